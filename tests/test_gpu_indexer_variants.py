"""Write-path variants of the MXFP4 lightning indexer ("DeepSeek V4" wiki
summary, section 基础设施: MXFP4 quantisation of the CSA indexer's QK path,
and FP4 -> FP8 dequantisation is lossless so FP8 machinery is reused):

  * CSA_FLAG_QI_BF16: the indexer takes bf16 queries and quantises them to
    MXFP4 inside the kernel.  Its MMA inputs are the bits csa_quantize would
    have stored, so its scores equal the stored-query path bit for bit, and
    the oracle's (its own quantiser, its own indexer) within the fp32 bound.
  * CSA_FLAG_INDEXER_FP8: the stored E2M1 codes are expanded to E4M3 (exact)
    and multiplied on the MXFP8 block-scaled MMA; every product is the same
    exact value, so the scores match the oracle within the same fp32 bound.

Shapes are the kernel's (64 heads x 128 dims); inputs span a wide exponent
range per key, block and head; the rows are ragged (every key eligible, a
partial row, none eligible); the many-row case gives every CTA more rows than
its query buffers, so buffer reuse is exercised."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from helpers import (both_stored, check_selection, down, orc_quantize, up)
from synth.workloads import WORKLOADS, draw_np

pytestmark = pytest.mark.gpu

HI, DI, M, W = 64, 128, 4, 128
VARIANTS = {"qi_bf16": K.FLAG_QI_BF16, "fp8": K.FLAG_INDEXER_FP8,
            "qi_bf16+fp8": K.FLAG_QI_BF16 | K.FLAG_INDEXER_FP8}


@pytest.fixture(autouse=True)
def _clean_status():
    K.csa_device_status(reset=True)
    yield
    assert K.csa_device_status(reset=True) == 0


def _bf16_round(a):
    """Host float32 -> nearest-even bf16 values (as float32) and their bits."""
    bits = oracle.f32_to_bf16(np.ascontiguousarray(a, np.float32))
    return (bits.astype(np.uint32) << 16).view(np.float32), bits


def _inputs(seed, batch, n_q, nb, wide):
    qv = synth.tensor_np(seed, "vq", (batch, n_q, HI, DI))
    kv_ = synth.tensor_np(seed, "vk", (batch, nb, DI))
    if wide:
        rng = np.random.default_rng(seed)
        qv = qv * np.exp2(rng.integers(-20, 21, (batch, n_q, HI, 1)))
        kv_ = kv_ * np.exp2(rng.integers(-40, 41, (batch, nb, 1)))
        kv_ = kv_ * np.repeat(np.exp2(rng.integers(-10, 11, (batch, nb, DI // 32))), 32, axis=2)
    # the queries are bf16 values, so both paths quantise the same numbers
    qv, q_bits = _bf16_round(qv)
    w = synth.tensor_np(seed, "vw", (batch, n_q, HI), std=0.1)
    return qv, q_bits, kv_.astype(np.float32), w


def _check_rows(got, qv, kv_, w, q_pos, rows):
    """Scores of the given (b, i) rows against the oracle, within 1e-5 of
    sum_h |w_h| |q_h| |k_j| (fp32 accumulation of exact products)."""
    nb = kv_.shape[1]
    for b, i in rows:
        qo = orc_quantize(qv[b, i].reshape(-1, DI), "mxfp4")
        ko = orc_quantize(kv_[b], "mxfp4")
        t = int(q_pos[b, i])
        ref = oracle.indexer(qo, w[b, i][None], ko, [t], HI, M, W)[0]
        ne = min(oracle.n_elig(t, M, W), nb)
        assert np.all(np.isnan(got[b, i, ne:])), "columns past n_elig must be untouched"
        if ne == 0:
            continue
        qdq = oracle.dequantize(qo)
        kdq = oracle.dequantize(ko)
        mag = (np.abs(w[b, i])[:, None] * np.linalg.norm(qdq, axis=1)[:, None] *
               np.linalg.norm(kdq[:ne], axis=1)[None, :]).sum(0)
        err = np.abs(got[b, i, :ne] - ref[:ne])
        assert (err <= 1e-5 * mag + 1e-30).all(), (b, i, err.max())


def _score(flags, qv, q_bits, kv_, w, q_pos):
    batch, n_q, nb = qv.shape[0], qv.shape[1], kv_.shape[1]
    p = K.params(M, W, 16, 1, 64, HI, DI, 1.0, idx_fmt=K.MXFP4, flags=flags)
    kd, _ = both_stored(kv_.reshape(-1, DI), "mxfp4")
    if flags & K.FLAG_QI_BF16:
        qd = K.Stored(K.BF16, up(q_bits.reshape(-1, DI), True))
    else:
        qd, _ = both_stored(qv.reshape(-1, DI), "mxfp4")
    scores = torch.full((batch, n_q, nb), float("nan"), device="cuda")
    K.indexer_score(p, batch, n_q, qd, up(w), kd, nb, up(q_pos), scores, nb)
    torch.cuda.synchronize()
    return down(scores)


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("wide", [False, True], ids=["normal", "wide_exponents"])
def test_indexer_variant_matches_oracle(variant, wide):
    batch, n_q, nb = 2, 3, 640
    qv, q_bits, kv_, w = _inputs(90 + wide, batch, n_q, nb, wide)
    q_pos = np.array([[M * nb + W + 5, M * 301 + W + 2, 7],
                      [M * nb + W, M * 129 + W + 3, M * 64 + W]], np.int64)
    got = _score(VARIANTS[variant], qv, q_bits, kv_, w, q_pos)
    _check_rows(got, qv, kv_, w, q_pos, [(b, i) for b in range(batch) for i in range(n_q)])
    base = _score(0, qv, q_bits, kv_, w, q_pos)
    if VARIANTS[variant] == K.FLAG_QI_BF16:
        # the same MMA on the same bits as the stored-query path
        assert np.array_equal(np.isnan(got), np.isnan(base))
        assert np.array_equal(got[~np.isnan(got)].view(np.uint32), base[~np.isnan(base)].view(np.uint32))


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_indexer_variant_many_rows(variant):
    """2,000 query rows of one 128-key step each: every CTA walks more rows
    than it has query buffers.  Sampled rows against the oracle; the fused
    query path bitwise against the stored-query path on every row."""
    batch, n_q, nb = 4, 500, 128
    qv, q_bits, kv_, w = _inputs(95, batch, n_q, nb, False)
    rng = np.random.default_rng(95)
    q_pos = rng.integers(0, M * nb + W + 40, size=(batch, n_q)).astype(np.int64)
    got = _score(VARIANTS[variant], qv, q_bits, kv_, w, q_pos)
    rows = [(b, i) for b in range(batch) for i in range(0, n_q, 37)] + [(batch - 1, n_q - 1)]
    _check_rows(got, qv, kv_, w, q_pos, rows)
    if VARIANTS[variant] == K.FLAG_QI_BF16:
        base = _score(0, qv, q_bits, kv_, w, q_pos)
        ok = ~np.isnan(base)
        assert np.array_equal(np.isnan(got), ~ok)
        assert np.array_equal(got[ok].view(np.uint32), base[ok].view(np.uint32))


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_csa_decode_with_indexer_variant(variant):
    """The whole decode step (indexer -> top-k -> sparse attention) with the
    variant's indexer: selections valid against the oracle's scores; with the
    fused query path, output and selection equal the default path's bits."""
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=3, n_ctx=8192, seed=17)
    B, H, d, k, nb = w.batch, w.H, w.d, w.k, w.n_blocks
    q_pos = np.array([8192, 6001, 4 * 300 + 128], np.int64)
    qv, q_bits = _bf16_round(draw_np(w, "qI"))
    kI = draw_np(w, "kI")
    wt = draw_np(w, "w")
    kv_d, _ = both_stored(draw_np(w, "kv").reshape(-1, d), "fp8")
    kI_d, _ = both_stored(kI.reshape(-1, DI), "mxfp4")
    q = up(draw_np(w, "q"), True)            # activations are drawn as bf16 bit patterns
    win = up(draw_np(w, "window"), True)
    sinks = up(draw_np(w, "sinks"))

    def run(flags):
        p = K.params(w.m, w.W, k, H, d, HI, DI, w.scale, K.BF16, K.FP8_S64, K.MXFP4, flags=flags)
        if flags & K.FLAG_QI_BF16:
            qd = K.Stored(K.BF16, up(q_bits.reshape(-1, DI), True))
        else:
            qd, _ = both_stored(qv.reshape(-1, DI), "mxfp4")
        out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((B, k), dtype=torch.int32, device="cuda")
        ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, B, 1, nb), dtype=torch.uint8, device="cuda")
        K.csa_decode(p, B, q, qd, up(wt), kv_d, kI_d, nb, win, w.W, up(q_pos - w.W + 1), up(q_pos),
                     sinks, out, sel, ws)
        torch.cuda.synchronize()
        return down(out), down(sel)

    out, sel = run(VARIANTS[variant])
    for b in range(B):
        t = int(q_pos[b])
        qo = orc_quantize(qv[b].reshape(-1, DI), "mxfp4")
        scores = oracle.indexer(qo, wt[b][None], orc_quantize(kI[b], "mxfp4"), [t], HI, w.m, w.W)[0]
        check_selection(sel[b], scores, min(oracle.n_elig(t, w.m, w.W), nb), k, what=f"seq {b}")
    if VARIANTS[variant] == K.FLAG_QI_BF16:
        out0, sel0 = run(0)
        assert np.array_equal(sel, sel0)
        assert np.array_equal(out, out0)


def test_indexer_variant_flags_rejected_off_the_mxfp4_path():
    """The variants belong to the MXFP4 tensor-core indexer: another index
    format is an argument error, an unsupported shape is refused."""
    batch, n_q, nb = 1, 1, 256
    scores = torch.zeros((batch, n_q, nb), device="cuda")
    q_pos = up(np.array([[M * nb + W]], np.int64))
    w = up(np.ones((batch, n_q, HI), np.float32))
    qb = torch.zeros((HI, DI), dtype=torch.bfloat16, device="cuda")
    kb = torch.zeros((nb, DI), dtype=torch.bfloat16, device="cuda")
    for flags in VARIANTS.values():
        p = K.params(M, W, 16, 1, 64, HI, DI, 1.0, idx_fmt=K.BF16, flags=flags)
        with pytest.raises(K.CsaError) as e:
            K.indexer_score(p, batch, n_q, K.Stored(K.BF16, qb), w, K.Stored(K.BF16, kb), nb, q_pos,
                            scores, nb)
        assert e.value.status == -1  # CSA_ERR_ARG
        # 32 index heads: no tensor-core MXFP4 indexer for this shape
        p = K.params(M, W, 16, 1, 64, 32, DI, 1.0, idx_fmt=K.MXFP4, flags=flags)
        kd = K.empty_stored(K.MXFP4, nb, DI)
        qd = K.Stored(K.BF16, torch.zeros((32, DI), dtype=torch.bfloat16, device="cuda"))
        with pytest.raises(K.CsaError) as e:
            K.indexer_score(p, batch, n_q, qd, up(np.ones((batch, n_q, 32), np.float32)), kd, nb, q_pos,
                            scores, nb)
        assert e.value.status in (-1, -3)  # CSA_ERR_ARG (no query scales) or CSA_ERR_UNSUPPORTED
