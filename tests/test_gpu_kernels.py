"""Per-kernel parity of the CUDA library against the CPU oracle.

Every test draws its inputs from the seeded generator, lets each side build
its own stored tensors with its own quantiser, runs the library through the
C ABI and the oracle on the CPU, and compares under the rules in helpers.py.
Sizes are small enough for the oracle to finish in seconds but span several
tiles and a ragged tail.
"""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from helpers import (FMT, act_dev, act_orc, assert_attention_close, assert_close_abs, assert_close_f32,
                     attention_bound_stored, bf16_values_match, both_stored, check_selection, down,
                     orc_quantize, quant_codes_match, sink_dominant, up)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    K.csa_device_status(reset=True)
    yield
    assert K.csa_device_status(reset=True) == 0


def _values(name, shape, seed=0, std=1.0):
    return synth.tensor_np(seed, name, shape, std)


# ---------------------------------------------------------------- quantisers
@pytest.mark.parametrize("rows,d", [(1, 64), (37, 512), (300, 128)])
def test_quantize_fp8_matches_oracle(rows, d):
    v = _values("qf8", (rows, d))
    v[0, :64] = 0.0
    if rows > 2:
        v[1, 3] = 1e5
        v[2] *= 1e-6
    g, o = both_stored(v, "fp8")
    assert np.array_equal(down(g.scales), o.scales)
    assert np.array_equal(down(g.data), o.data)


@pytest.mark.parametrize("rows,d", [(1, 64), (33, 128), (300, 512)])
def test_quantize_mxfp4_matches_oracle(rows, d):
    v = _values("qf4", (rows, d))
    v[0, :32] = 0.0
    if rows > 2:
        v[1] *= 1000.0
        v[2, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4, np.float32)
    g, o = both_stored(v, "mxfp4")
    assert np.array_equal(down(g.scales), o.scales)
    assert np.array_equal(down(g.data), o.data)


def test_quantize_bf16_matches_oracle():
    v = _values("qbf", (50, 128)) * 7
    g, o = both_stored(v, "bf16")
    assert np.array_equal(down(g.data), o.data)


# ------------------------------------------------------------------- pooling
@pytest.mark.parametrize("act,m,d,n_blocks,out", [
    ("f32", 4, 64, 256, "f32"),
    ("bf16", 4, 512, 97, "f32"),
    ("bf16", 128, 512, 5, "f32"),
    ("f32", 4, 128, 33, "f32"),
    # m a multiple of 16: the staged kernel (bulk copies through shared memory)
    ("f32", 128, 512, 7, "f32"),
    ("bf16", 32, 256, 300, "f32"),        # more rows than CTAs
    ("bf16", 16, 64, 9, "f32"),
])
def test_compress_f32_out(act, m, d, n_blocks, out):
    n = m * n_blocks
    x = synth.tensor_np(1, "cx", (n, d), dtype=act)
    z = synth.tensor_np(1, "cz", (n, d), dtype=act)
    B = synth.tensor_np(1, "cb", (m, d), std=0.1)
    p = K.params(m, 0, 1, 1, d, 1, 32, 1.0, act_fmt=FMT[act])
    st = K.empty_stored(K.F32, n_blocks, d)
    K.csa_compress(p, d, act_dev(x, act), act_dev(z, act), up(B), n, st)
    ref = oracle.compress(act_orc(x, act), act_orc(z, act), B, m)
    assert_close_f32(down(st.data), ref, 1e-5, "pooled entries")


@pytest.mark.parametrize("act,m,d,n_blocks,fmt", [
    ("bf16", 4, 512, 64, "fp8"),
    ("bf16", 128, 512, 6, "fp8"),
    ("bf16", 4, 512, 40, "bf16"),
    ("f32", 4, 128, 70, "mxfp4"),
    ("bf16", 128, 512, 600, "fp8"),       # staged kernel, several rows per CTA
    ("bf16", 16, 128, 50, "mxfp4"),
    ("f32", 64, 512, 5, "bf16"),
])
def test_compress_quantised_out(act, m, d, n_blocks, fmt):
    n = m * n_blocks
    x = synth.tensor_np(2, "cx", (n, d), dtype=act)
    z = synth.tensor_np(2, "cz", (n, d), dtype=act)
    B = synth.tensor_np(2, "cb", (m, d), std=0.1)
    p = K.params(m, 0, 1, 1, d, 1, 32, 1.0, act_fmt=FMT[act])
    st = K.empty_stored(FMT[fmt], n_blocks, d)
    K.csa_compress(p, d, act_dev(x, act), act_dev(z, act), up(B), n, st)
    pre = oracle.compress(act_orc(x, act), act_orc(z, act), B, m)
    o = orc_quantize(pre, fmt)
    if fmt == "bf16":
        # both sides round their own fp32 value to bf16: values may differ
        # only on a rounding boundary (within the fp32 rule of it)
        assert bf16_values_match(down(st.data), o.data, pre) == 0
        return
    gs = down(st.scales)
    assert_close_f32(gs, o.scales, 1e-5, "scales")
    if fmt == "fp8":
        per_el = np.repeat(o.scales, 64, axis=1)
        bad = quant_codes_match(down(st.data), o.data, pre, per_el, "fp8")
    else:
        assert np.array_equal(gs, o.scales)
        per_el = np.repeat(2.0 ** (o.scales.astype(np.float64) - 127), 32, axis=1)
        g_codes = down(st.data)
        def unpack(a):
            a = a.astype(np.uint8)
            return np.stack([a & 15, a >> 4], -1).reshape(a.shape[0], -1)
        bad = quant_codes_match(unpack(g_codes), unpack(o.data), pre, per_el, "mxfp4")
    assert bad == 0


# ------------------------------------------------------------------- indexer
@pytest.mark.parametrize("idx,HI,dI,n_q,nb,m,W", [
    ("f32", 4, 32, 40, 256, 4, 64),
    ("bf16", 64, 128, 12, 700, 4, 128),
    ("bf16", 64, 128, 13, 300, 4, 128),
    ("bf16", 64, 128, 2, 300, 4, 128),
    ("mxfp4", 64, 128, 3, 2100, 4, 128),
])
def test_indexer_matches_oracle(idx, HI, dI, n_q, nb, m, W):
    batch = 2
    qv = synth.tensor_np(3, "iq", (batch, n_q, HI, dI), dtype="f32" if idx != "bf16" else "bf16")
    kv_ = synth.tensor_np(3, "ik", (batch, nb, dI), dtype="f32" if idx != "bf16" else "bf16")
    w = synth.tensor_np(3, "iw", (batch, n_q, HI), std=0.1)
    rng = np.random.default_rng(3)
    q_pos = rng.integers(0, m * nb + W + 50, size=(batch, n_q)).astype(np.int64)
    q_pos[0, 0] = m * nb + W + 10      # every block eligible
    q_pos[1, 0] = 3                    # none eligible
    p = K.params(m, W, 16, 1, 64, HI, dI, 1.0, idx_fmt=FMT[idx])
    if idx == "bf16":
        qd = K.Stored(K.BF16, up(qv, True))
        kd = K.Stored(K.BF16, up(kv_, True))
        qo = [oracle.Stored(oracle.BF16, qv[b].reshape(-1, dI)) for b in range(batch)]
        ko = [oracle.Stored(oracle.BF16, kv_[b]) for b in range(batch)]
    else:
        qd, _ = both_stored(qv.reshape(-1, dI), idx)
        kd, _ = both_stored(kv_.reshape(-1, dI), idx)
        qo = [orc_quantize(qv[b].reshape(-1, dI), idx) for b in range(batch)]
        ko = [orc_quantize(kv_[b], idx) for b in range(batch)]
    scores = torch.full((batch, n_q, nb), float("nan"), device="cuda")
    K.indexer_score(p, batch, n_q, qd, up(w), kd, nb, up(q_pos), scores, nb)
    got = down(scores)
    for b in range(batch):
        ref = oracle.indexer(qo[b], w[b], ko[b], q_pos[b], HI, m, W)
        qdq = oracle.dequantize(qo[b]).reshape(n_q, HI, dI)
        kdq = oracle.dequantize(ko[b])
        for i in range(n_q):
            ne = min(oracle.n_elig(int(q_pos[b, i]), m, W), nb)
            assert np.all(np.isnan(got[b, i, ne:])), "columns past n_elig must be untouched"
            if ne == 0:
                continue
            # fp32 accumulation bound: 1e-5 of sum_h |w_h| |q_h| |k_j|
            mag = (np.abs(w[b, i])[:, None] * np.linalg.norm(qdq[i], axis=1)[:, None] *
                   np.linalg.norm(kdq[:ne], axis=1)[None, :]).sum(0)
            err = np.abs(got[b, i, :ne] - ref[i, :ne])
            assert (err <= 1e-5 * mag + 1e-30).all(), (b, i, err.max())


# --------------------------------------------------------------------- top-k
# Up to 32,768 scores: the sampled-threshold kernel (1, 4 or 8 CTAs per row);
# longer rows: a cluster per row (few rows) or one CTA per row reading the
# row from global memory; many rows (>= 296) of up to 2,048 scores: one warp
# per row; of up to 4,096: one CTA per row in shared memory.
@pytest.mark.parametrize("n,k,rows", [
    (50, 8, 6), (2015, 512, 6), (32736, 512, 6), (5000, 1024, 6), (60000, 1024, 6),
    (2015, 512, 48), (32736, 512, 48),
    (70000, 1024, 6), (250000, 1024, 6),
    (60000, 1024, 40), (300000, 512, 6),
    (2016, 512, 300), (2048, 1024, 301), (700, 64, 400),                              # warp per row
    (4000, 512, 300),                                                                  # shared memory
])
def test_topk_matches_oracle_exactly(n, k, rows):
    s = synth.tensor_np(4, "ts", (rows, n))
    s[1] = np.round(s[1] * 2) / 2          # many exact ties
    s[2, ::3] = 0.0
    s[2, 1::3] = -0.0                      # -0 and +0 are equal
    s[3] = 0.25                            # all equal
    m, W = 4, 128
    q_pos = np.full(rows, m * n + W + 3, np.int64)
    q_pos[4] = m * (k // 2) + W           # n_elig < k
    q_pos[5] = m * k + W                  # n_elig == k
    p = K.params(m, W, k, 1, 64, 1, 32, 1.0)
    idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    K.topk_select(p, 1, rows, up(s), n, n, up(q_pos), idx)
    ref = oracle.topk(s, q_pos, k, m, W)
    assert np.array_equal(down(idx), ref)


# ----------------------------------------------------------------- attention
def _attn_case(act, kvf, H, d, batch, n_q, n_ent, W, k, m, seed, scale):
    qv = synth.tensor_np(seed, "aq", (batch, n_q, H, d), dtype=act)
    ent = synth.tensor_np(seed, "akv", (batch, n_ent, d))
    n_raw = W + 40
    raw = synth.tensor_np(seed, "araw", (batch, n_raw, d), dtype=act)
    sinks = synth.tensor_np(seed, "asink", (H,))
    rng = np.random.default_rng(seed)
    t_hi = m * n_ent + W + 20
    q_pos = rng.integers(0, t_hi, size=(batch, n_q)).astype(np.int64)
    q_pos[:, 0] = t_hi
    raw_pos0 = np.maximum(q_pos.max(1) - n_raw + 1, 0).astype(np.int64)
    raw_pos0[0] = max(0, t_hi - W - 10)
    return qv, ent, raw, n_raw, sinks, q_pos, raw_pos0


# 2 x 12 and 2 x 20 query rows split each row 6 and 3 ways on the tensor-core
# path, where the splits of a row form a cluster and combine in the kernel
# (2 x 9, 2 x 10 and 2 x 13 rows: 8, 7 and 5 splits); 6 rows split 10 ways
# and use the separate combine kernel.
@pytest.mark.parametrize("act,kvf,H,d,n_q,n_ent,W,k,m", [
    ("f32", "f32", 8, 64, 20, 256, 64, 16, 4),
    ("bf16", "fp8", 64, 512, 3, 700, 128, 512, 4),
    ("bf16", "fp8", 64, 512, 9, 700, 128, 512, 4),
    ("bf16", "fp8", 64, 512, 10, 700, 128, 512, 4),
    ("bf16", "fp8", 64, 512, 13, 700, 128, 512, 4),
    ("bf16", "fp8", 64, 512, 12, 700, 128, 512, 4),
    ("bf16", "fp8", 64, 512, 20, 400, 128, 256, 4),
    ("bf16", "bf16", 64, 512, 4, 300, 128, 64, 4),
    ("bf16", "bf16", 64, 512, 3, 700, 128, 512, 4),
    ("bf16", "bf16", 64, 512, 160, 900, 128, 512, 4),
])
def test_sparse_attention_matches_oracle(act, kvf, H, d, n_q, n_ent, W, k, m):
    batch, seed, scale = 2, 5, 1 / math.sqrt(d)
    qv, ent, raw, n_raw, sinks, q_pos, raw_pos0 = _attn_case(act, kvf, H, d, batch, n_q, n_ent, W, k, m, seed, scale)
    rng = np.random.default_rng(seed + 1)
    idx = np.full((batch, n_q, k), -1, np.int32)
    for b in range(batch):
        for i in range(n_q):
            ne = min(oracle.n_elig(int(q_pos[b, i]), m, W), n_ent)
            c = np.sort(rng.permutation(ne)[:min(k, ne)])
            idx[b, i, :len(c)] = c
    kd, _ = both_stored(ent.reshape(-1, d), kvf)
    p = K.params(m, W, k, H, d, 1, 32, scale, act_fmt=FMT[act], kv_fmt=FMT[kvf])
    out = torch.empty((batch, n_q, H, d), dtype=torch.float32 if act == "f32" else torch.bfloat16,
                      device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_SPARSE_ATTN, batch, n_q, 0), dtype=torch.uint8,
                     device="cuda")
    K.sparse_mqa_attn(p, batch, n_q, act_dev(qv, act), kd, n_ent, up(idx), act_dev(raw, act),
                      n_raw, up(raw_pos0), up(q_pos), up(sinks), out, ws)
    got = down(out.float())
    for b in range(batch):
        args = (act_orc(qv[b], act), orc_quantize(ent[b], kvf), idx[b], act_orc(raw[b], act),
                int(raw_pos0[b]))
        ref = oracle.attention(*args, sinks, q_pos[b], H, m, W, scale)
        if act == "f32":
            assert_close_f32(got[b], ref, 1e-5, f"seq {b}")
        else:
            bound = attention_bound_stored(*args, sinks, q_pos[b], H, m, W, scale)
            assert_attention_close(got[b], ref, bound, f"seq {b}")


@pytest.mark.parametrize("act,kvf,H,d,n_q,n_ent,W,m", [
    ("f32", "f32", 8, 64, 10, 300, 64, 4),
    ("bf16", "fp8", 64, 512, 2, 1500, 128, 128),
    ("bf16", "bf16", 64, 512, 2, 1500, 128, 128),
    ("bf16", "bf16", 64, 512, 3, 333, 128, 4),
])
def test_hca_attention_matches_oracle(act, kvf, H, d, n_q, n_ent, W, m):
    batch, seed, scale = 2, 6, 1 / math.sqrt(d)
    qv, ent, raw, n_raw, sinks, q_pos, raw_pos0 = _attn_case(act, kvf, H, d, batch, n_q, n_ent, W, 0, m, seed, scale)
    kd, _ = both_stored(ent.reshape(-1, d), kvf)
    p = K.params(m, W, 1, H, d, 1, 32, scale, act_fmt=FMT[act], kv_fmt=FMT[kvf])
    out = torch.empty((batch, n_q, H, d), dtype=torch.float32 if act == "f32" else torch.bfloat16,
                      device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, batch, n_q, n_ent), dtype=torch.uint8,
                     device="cuda")
    K.hca_attn(p, batch, n_q, act_dev(qv, act), kd, n_ent, act_dev(raw, act), n_raw, up(raw_pos0),
               up(q_pos), up(sinks), out, ws)
    got = down(out.float())
    for b in range(batch):
        args = (act_orc(qv[b], act), orc_quantize(ent[b], kvf), None, act_orc(raw[b], act),
                int(raw_pos0[b]))
        ref = oracle.attention(*args, sinks, q_pos[b], H, m, W, scale)
        if act == "f32":
            assert_close_f32(got[b], ref, 1e-5, f"seq {b}")
        else:
            bound = attention_bound_stored(*args, sinks, q_pos[b], H, m, W, scale)
            assert_attention_close(got[b], ref, bound, f"seq {b}")


# Rows whose outcome hinges on the sink and on each item: sink logits 2 above
# every attended logit (the sink dominates the denominators), and positions
# with few items: t < W (t + 1 raw tokens, no pooled entry) and t >= W with at
# most three visible pooled blocks.  For each case the oracle also computes the
# two mistakes these rows are there to catch -- the sink left out, and the
# window one token short (or the query's own token left out) -- and the test
# first checks that each of those misses the tolerance, so that a kernel
# making it would fail.
@pytest.mark.parametrize("kvf,dense,n_splits_hint", [
    ("fp8", False, "few rows: splits combined in the cluster"),
    ("bf16", False, "bf16 entries gathered by the converters"),
    ("fp8", True, "HCA: dense entries"),
])
def test_attention_sink_dominant_and_few_item_rows(kvf, dense, n_splits_hint):
    H, d, m, W, k, seed = 64, 512, 4, 128, 16, 31
    scale = 1 / math.sqrt(d)
    n_ent, batch = 3, 2
    # sequence 0: positions below the window; sequence 1: t >= W with <= 3 blocks
    q_pos = np.array([[0, 1, 5, 17, 40, 126], [W, W + 1, W + m, W + 2 * m + 1, W + 3 * m, W + 3 * m + 3]],
                     np.int64)
    n_q = q_pos.shape[1]
    n_raw = W + 3 * m + 4
    raw_pos0 = np.zeros(batch, np.int64)
    qv = synth.tensor_np(seed, "sq", (batch, n_q, H, d), dtype="bf16")
    ent = synth.tensor_np(seed, "skv", (batch, n_ent, d))
    raw = synth.tensor_np(seed, "sraw", (batch, n_raw, d), dtype="bf16")
    idx = np.full((batch, n_q, k), -1, np.int32)
    for b in range(batch):
        for i in range(n_q):
            ne = min(oracle.n_elig(int(q_pos[b, i]), m, W), n_ent)
            idx[b, i, :ne] = np.arange(ne)
    kd, _ = both_stored(ent.reshape(-1, d), kvf)
    orc_in = [(act_orc(qv[b], "bf16"), orc_quantize(ent[b], kvf), None if dense else idx[b],
               act_orc(raw[b], "bf16"), 0) for b in range(batch)]
    sinks = np.max([sink_dominant(*orc_in[b], q_pos[b], H, m, W, scale) for b in range(batch)], axis=0)
    p = K.params(m, W, k, H, d, 1, 32, scale, act_fmt=K.BF16, kv_fmt=FMT[kvf])
    out = torch.empty((batch, n_q, H, d), dtype=torch.bfloat16, device="cuda")
    args = (p, batch, n_q, act_dev(qv, "bf16"), kd, n_ent)
    tail = (act_dev(raw, "bf16"), n_raw, up(raw_pos0), up(q_pos), up(sinks), out)
    if dense:
        ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, batch, n_q, n_ent), dtype=torch.uint8,
                         device="cuda")
        K.hca_attn(*args, *tail, ws)
    else:
        ws = torch.empty(K.csa_workspace_size(p, K.OP_SPARSE_ATTN, batch, n_q, 0), dtype=torch.uint8,
                         device="cuda")
        K.sparse_mqa_attn(*args, up(idx), *tail, ws)
    got = down(out.float())
    for b in range(batch):
        ref = oracle.attention(*orc_in[b], sinks, q_pos[b], H, m, W, scale)
        bound = attention_bound_stored(*orc_in[b], sinks, q_pos[b], H, m, W, scale)
        # the planted mistakes (on the CPU) miss the tolerance on every row
        no_sink = oracle.attention(*orc_in[b], np.full(H, -np.inf, np.float32), q_pos[b], H, m, W, scale)
        assert ((np.abs(no_sink - ref) > bound).any(axis=(1, 2))).all()
        if b == 0:
            short = oracle.attention(*orc_in[b], sinks, q_pos[b] - 1, H, m, W, scale)  # own token left out
            rows = q_pos[b] >= 1
        else:
            short = oracle.attention(*orc_in[b], sinks, q_pos[b], H, m, W - 1, scale)
            rows = np.ones(n_q, bool)
        assert ((np.abs(short - ref) > bound).any(axis=(1, 2)))[rows].all()
        assert_attention_close(got[b], ref, bound, f"seq {b}")


def test_out_of_range_index_is_flagged_not_read():
    H, d, m, W, k = 8, 64, 4, 4, 4
    p = K.params(m, W, k, H, d, 1, 32, 0.125, act_fmt=K.F32, kv_fmt=K.F32)
    q = torch.randn(1, 1, H, d, device="cuda")
    kv = K.Stored(K.F32, torch.randn(10, d, device="cuda"))
    idx = torch.tensor([[[0, 3, 1 << 20, -1]]], dtype=torch.int32, device="cuda")
    raw = torch.randn(1, 8, d, device="cuda")
    out = torch.empty(1, 1, H, d, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_SPARSE_ATTN, 1, 1, 0), dtype=torch.uint8, device="cuda")
    K.sparse_mqa_attn(p, 1, 1, q, kv, 10, idx, raw, 8, up(np.array([0])), up(np.array([7])), None, out, ws)
    assert K.csa_device_status(reset=True) == K.DEV_BAD_INDEX
    assert torch.isfinite(out).all()


def test_mxfp4_indexer_exact_across_block_exponents():
    """The block-scaled tensor-core indexer applies E8M0 exponents in the MMA
    itself, so keys and queries whose blocks span a wide exponent range (per
    key 2^-40 .. 2^40, per block a further 2^+-10, per query head 2^+-20) still
    match the oracle within the fp32 accumulation bound, and nothing is flagged."""
    HI, dI, nb, m, W, batch, n_q = 64, 128, 640, 4, 128, 2, 2
    rng = np.random.default_rng(81)
    qv = synth.tensor_np(8, "rq", (batch, n_q, HI, dI))
    qv = qv * np.exp2(rng.integers(-20, 21, (batch, n_q, HI, 1)))
    kv_ = synth.tensor_np(8, "rk", (batch, nb, dI))
    kv_ = kv_ * np.exp2(rng.integers(-40, 41, (batch, nb, 1)))
    kv_ = kv_ * np.repeat(np.exp2(rng.integers(-10, 11, (batch, nb, dI // 32))), 32, axis=2)
    w = synth.tensor_np(8, "rw", (batch, n_q, HI), std=0.1)
    q_pos = np.array([[m * nb + W, m * 300 + W + 3], [m * nb + W + 7, m * 129 + W]], np.int64)
    p = K.params(m, W, 16, 1, 64, HI, dI, 1.0, idx_fmt=K.MXFP4)
    qd, _ = both_stored(qv.reshape(-1, dI).astype(np.float32), "mxfp4")
    kd, _ = both_stored(kv_.reshape(-1, dI).astype(np.float32), "mxfp4")
    scores = torch.full((batch, n_q, nb), float("nan"), device="cuda")
    K.indexer_score(p, batch, n_q, qd, up(w), kd, nb, up(q_pos), scores, nb)
    assert K.csa_device_status(reset=True) == 0
    got = down(scores)
    for b in range(batch):
        qo = orc_quantize(qv[b].reshape(-1, dI).astype(np.float32), "mxfp4")
        ko = orc_quantize(kv_[b].astype(np.float32), "mxfp4")
        ref = oracle.indexer(qo, w[b], ko, q_pos[b], HI, m, W)
        qdq = oracle.dequantize(qo).reshape(n_q, HI, dI)
        kdq = oracle.dequantize(ko)
        for i in range(n_q):
            ne = min(oracle.n_elig(int(q_pos[b, i]), m, W), nb)
            mag = (np.abs(w[b, i])[:, None] * np.linalg.norm(qdq[i], axis=1)[:, None] *
                   np.linalg.norm(kdq[:ne], axis=1)[None, :]).sum(0)
            err = np.abs(got[b, i, :ne] - ref[i, :ne])
            assert (err <= 1e-5 * mag + 1e-30).all(), (b, i, err.max())


# Window-only attention (the MTP block): few-item rows (t < W) in one sequence,
# full windows in the other, with and without sink-dominant logits; the bf16
# tensor-core path and the fp32 CUDA-core path.
@pytest.mark.parametrize("act,H,d,W,sink_shift", [
    ("bf16", 64, 512, 128, None),
    ("bf16", 64, 512, 128, 2.0),
    ("f32", 8, 64, 64, None),
])
def test_window_attn_matches_oracle(act, H, d, W, sink_shift):
    seed, batch = 41, 2
    scale = 1 / math.sqrt(d)
    q_pos = np.array([[0, 1, 4, 17, 60, W - 1], [W + 300, W + 301, W + 350, W + 400, W + 433, W + 439]],
                     np.int64)
    n_q = q_pos.shape[1]
    raw_pos0 = np.array([0, W + 300 - W + 1], np.int64)
    n_raw = int(max(q_pos[b].max() - raw_pos0[b] + 1 for b in range(batch)))
    qv = synth.tensor_np(seed, "wq", (batch, n_q, H, d), dtype=act)
    raw = synth.tensor_np(seed, "wraw", (batch, n_raw, d), dtype=act)
    empty = oracle.Stored(oracle.F32, np.zeros((0, d), np.float32))
    orc_in = [(act_orc(qv[b], act), empty, None, act_orc(raw[b], act), int(raw_pos0[b])) for b in range(batch)]
    sinks = synth.tensor_np(seed, "wsink", (H,))
    if sink_shift is not None:
        sinks = np.max([sink_dominant(*orc_in[b], q_pos[b], H, 4, W, scale, sink_shift)
                        for b in range(batch)], axis=0)
    p = K.params(4, W, 1, H, d, 1, 32, scale, act_fmt=FMT[act], kv_fmt=FMT[act] if act == "f32" else K.FP8_S64)
    out = torch.empty((batch, n_q, H, d), dtype=torch.float32 if act == "f32" else torch.bfloat16, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_WINDOW_ATTN, batch, n_q, 0), dtype=torch.uint8, device="cuda")
    K.window_attn(p, batch, n_q, act_dev(qv, act), act_dev(raw, act), n_raw, up(raw_pos0), up(q_pos),
                  up(sinks), out, ws)
    got = down(out.float())
    for b in range(batch):
        ref = oracle.attention(*orc_in[b], sinks, q_pos[b], H, 4, W, scale)
        if act == "f32":
            assert_close_f32(got[b], ref, 1e-5, f"seq {b}")
        else:
            bound = attention_bound_stored(*orc_in[b], sinks, q_pos[b], H, 4, W, scale)
            assert_attention_close(got[b], ref, bound, f"seq {b}")
