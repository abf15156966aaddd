"""End-to-end parity of the fused entry points (csa_decode, csa_prefill, and the
HCA decode path compress -> hca_attn) against the oracle, on reduced copies of
the workloads with ragged positions and the edge cases of the method."""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from helpers import (FMT, act_dev, act_orc, assert_attention_close, assert_close_abs, assert_close_f32,
                     attention_bound_stored, both_stored, check_selection, down, orc_quantize,
                     sink_dominant, up)
from synth.workloads import WORKLOADS, draw_np

pytestmark = pytest.mark.gpu


def _threads():
    """Oracle threads for the larger checks (independent query rows)."""
    import os
    return max(1, len(os.sched_getaffinity(0)))


@pytest.fixture(autouse=True)
def _clean_status():
    K.csa_device_status(reset=True)
    yield
    assert K.csa_device_status(reset=True) == 0


def run_decode_case(w, q_pos, check_rows=None, sink_shift=None):
    """CSA decode through csa_decode; returns (out, sel) on the host plus the
    oracle-side stored inputs for checking."""
    B, H, d, HI, dI, m, W, k = w.batch, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = w.n_blocks
    q = draw_np(w, "q")
    qI = draw_np(w, "qI")
    wt = draw_np(w, "w")
    kv = draw_np(w, "kv")
    kI = draw_np(w, "kI")
    win = draw_np(w, "window")
    sinks = draw_np(w, "sinks")
    p = K.params(m, W, k, H, d, HI, dI, w.scale, FMT[w.act], FMT[w.kv], FMT[w.idx])
    kv_d, _ = both_stored(kv.reshape(-1, d), w.kv)
    kI_d, _ = both_stored(kI.reshape(-1, dI), w.idx)
    qI_d, _ = both_stored(qI.reshape(-1, dI), w.idx)
    q_pos = np.asarray(q_pos, np.int64)
    raw_pos0 = q_pos - W + 1
    if sink_shift is not None:
        # sinks above every logit any selection could contain (all visible blocks)
        sinks = np.max([sink_dominant(act_orc(q[b], w.act), orc_quantize(kv[b], w.kv), None,
                                      act_orc(win[b], w.act), int(raw_pos0[b]), [int(q_pos[b])],
                                      H, m, W, w.scale, sink_shift) for b in range(B)], axis=0)
    out = torch.empty((B, H, d), dtype=torch.bfloat16 if w.act == "bf16" else torch.float32,
                      device="cuda")
    sel = torch.empty((B, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, B, 1, nb), dtype=torch.uint8, device="cuda")
    K.csa_decode(p, B, act_dev(q, w.act), qI_d, up(wt), kv_d, kI_d, nb, act_dev(win, w.act), W,
                 up(raw_pos0), up(q_pos), up(sinks), out, sel, ws)
    got, got_sel = down(out.float()), down(sel)
    rows = range(B) if check_rows is None else check_rows
    for b in rows:
        t = int(q_pos[b])
        qI_o = orc_quantize(qI[b].reshape(-1, dI), w.idx)
        kI_o = orc_quantize(kI[b], w.idx)
        kv_o = orc_quantize(kv[b], w.kv)
        scores = oracle.indexer(qI_o, wt[b][None], kI_o, [t], HI, m, W)[0]
        ne = min(oracle.n_elig(t, m, W), nb)
        check_selection(got_sel[b], scores, ne, k, what=f"seq {b}")
        # output against the oracle's attention over the library's (valid) selection
        args = (act_orc(q[b], w.act), kv_o, got_sel[b][None], act_orc(win[b], w.act), t - W + 1)
        ref = oracle.attention(*args, sinks, [t], H, m, W, w.scale)[0]
        if w.act == "f32":
            assert_close_f32(got[b], ref, 1e-5, f"seq {b}")
        else:
            bound = attention_bound_stored(*args, sinks, [t], H, m, W, w.scale)[0]
            assert_attention_close(got[b], ref, bound, f"seq {b}")
    return got, got_sel


def test_csa_decode_reduced_ragged():
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=4, n_ctx=8192, seed=11)
    # ragged: full context, partial, fewer eligible blocks than k, none eligible
    q_pos = [8192, 8000, 4 * 300 + 128, 50]
    run_decode_case(w, q_pos)


def test_csa_decode_sink_dominant():
    """Sink logits 2 above every attended logit: the outputs shrink by about
    e^-2 and a mishandled sink fails both matching rules."""
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=3, n_ctx=4096, seed=14)
    run_decode_case(w, [4096, 2500, 4 * 200 + 128], sink_shift=2.0)


def test_csa_decode_degenerate_all_blocks_no_window():
    """k >= n_elig with W = 0: decode reduces to dense attention over the
    eligible entries (the oracle check uses the dense routine)."""
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=2, n_ctx=1024, k=512, W=0, seed=12)
    q_pos = [1024, 900]
    got, sel = run_decode_case(w, q_pos)
    for b, t in enumerate(q_pos):
        ne = oracle.n_elig(t, w.m, 0)
        assert list(sel[b, :ne]) == list(range(ne)) and np.all(sel[b, ne:] == -1)


def test_csa_prefill_tiny_fp32_full():
    """The whole fp32 prefill workload (T = 1024), every query checked."""
    w = WORKLOADS["csa_prefill_1k_fp32"]
    _run_prefill(w, check_every=1)


def test_csa_prefill_bf16_reduced():
    w = WORKLOADS["csa_prefill_8k_bf16"].with_(n_ctx=640, seed=3)
    _run_prefill(w, check_every=7)


def _run_prefill(w, check_every):
    B, T, H, d, HI, dI, m, W, k = w.batch, w.n_ctx, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = T // m
    x, z, bias = draw_np(w, "x"), draw_np(w, "z"), draw_np(w, "bias")
    q, qI, wt = draw_np(w, "q"), draw_np(w, "qI"), draw_np(w, "w")
    kI, sinks = draw_np(w, "kI"), draw_np(w, "sinks")
    p = K.params(m, W, k, H, d, HI, dI, w.scale, FMT[w.act], FMT[w.kv], FMT[w.idx])
    if w.idx == "bf16":
        qI_d, kI_d = K.Stored(K.BF16, up(qI, True)), K.Stored(K.BF16, up(kI, True))
    else:
        qI_d, _ = both_stored(qI.reshape(-1, dI), w.idx)
        kI_d, _ = both_stored(kI.reshape(-1, dI), w.idx)
    kv_d = K.empty_stored(FMT[w.kv], B * nb, d)
    out = torch.empty((B, T, H, d), dtype=torch.bfloat16 if w.act == "bf16" else torch.float32,
                      device="cuda")
    sel = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_PREFILL, B, T, nb), dtype=torch.uint8, device="cuda")
    K.csa_prefill(p, B, T, 0, act_dev(x, w.act), T, 0, act_dev(z, w.act), up(bias),
                  act_dev(q, w.act), qI_d, up(wt), kv_d, kI_d, nb, up(sinks), out, sel, ws)
    got, got_sel = down(out.float()), down(sel)
    for b in range(B):
        pooled = oracle.compress(act_orc(x[b], w.act), act_orc(z[b], w.act), bias, m)
        kv_o = orc_quantize(pooled, w.kv)
        if w.idx == "bf16":
            qI_o = oracle.Stored(oracle.BF16, qI[b].reshape(-1, dI))
            kI_o = oracle.Stored(oracle.BF16, kI[b])
        else:
            qI_o, kI_o = orc_quantize(qI[b].reshape(-1, dI), w.idx), orc_quantize(kI[b], w.idx)
        rows = np.arange(0, T, check_every)
        rows = np.unique(np.concatenate([rows, [T - 1]]))
        qI_rows = oracle.Stored(qI_o.fmt, qI_o.data.reshape(T, HI, -1)[rows].reshape(-1, qI_o.data.shape[-1]),
                                None if qI_o.scales is None else
                                qI_o.scales.reshape(T, HI, -1)[rows].reshape(-1, qI_o.scales.shape[-1]), dI)
        scores = oracle.indexer(qI_rows, wt[b][rows], kI_o, rows, HI, m, W)
        for a, t in enumerate(rows):
            ne = min(oracle.n_elig(int(t), m, W), nb)
            check_selection(got_sel[b, t], scores[a], ne, k, what=f"seq {b} t {t}")
        q_rows = q[b][rows]
        args = (act_orc(q_rows.reshape(-1, d), w.act), kv_o, got_sel[b][rows], act_orc(x[b], w.act), 0)
        ref = oracle.attention(*args, sinks, rows, H, m, W, w.scale, n_threads=_threads())
        if w.act == "f32":
            assert_close_f32(got[b][rows], ref, 1e-5, f"prefill seq {b}")
        else:
            bound = attention_bound_stored(*args, sinks, rows, H, m, W, w.scale)
            assert_attention_close(got[b][rows], ref, bound, f"prefill seq {b}")


def test_hca_decode_reduced():
    """HCA decode: pool the context at m' = 128 into FP8 entries (library
    compress), then dense attention over every visible entry + window + sink."""
    w = WORKLOADS["hca_decode_1m_b8"].with_(batch=2, n_ctx=1 << 16, seed=13)
    _run_hca(w, check_batches=[0, 1])


def _run_hca(w, check_batches, draw_on_device=False):
    B, N, H, d, m, W = w.batch, w.n_ctx, w.H, w.d, w.m, w.W
    nb = N // m
    p = K.params(m, W, 1, H, d, 1, 32, w.scale, FMT[w.act], FMT[w.kv], K.MXFP4)
    if draw_on_device:
        from synth.workloads import draw_torch
        x_d, z_d = draw_torch(w, "x"), draw_torch(w, "z")
    else:
        x_d, z_d = act_dev(draw_np(w, "x"), w.act), act_dev(draw_np(w, "z"), w.act)
    bias = draw_np(w, "bias")
    kv_d = K.empty_stored(FMT[w.kv], B * nb, d)
    K.csa_compress(p, d, x_d, z_d, up(bias), B * N, kv_d)
    x_new, q, sinks = draw_np(w, "x_new"), draw_np(w, "q"), draw_np(w, "sinks")
    # window buffer: the last W-1 context tokens and the new token
    win_d = torch.cat([x_d[:, N - W + 1:], act_dev(x_new, w.act)[:, None]], dim=1).contiguous()
    q_pos = np.full(B, N, np.int64)
    raw_pos0 = q_pos - W + 1
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, B, 1, nb), dtype=torch.uint8, device="cuda")
    K.hca_attn(p, B, 1, act_dev(q, w.act), kv_d, nb, win_d, W, up(raw_pos0), up(q_pos), up(sinks), out, ws)
    got = down(out.float())
    for b in check_batches:
        xb = down(x_d[b]) if draw_on_device else draw_np(w, "x", b)
        zb = down(z_d[b]) if draw_on_device else draw_np(w, "z", b)
        pooled = oracle.compress(act_orc(xb, w.act), act_orc(zb, w.act), bias, m)
        kv_o = orc_quantize(pooled, w.kv)
        win = np.concatenate([xb[N - W + 1:], x_new[b][None]])
        args = (act_orc(q[b], w.act), kv_o, None, act_orc(win, w.act), N - W + 1)
        ref = oracle.attention(*args, sinks, [N], H, m, W, w.scale)[0]
        bound = attention_bound_stored(*args, sinks, [N], H, m, W, w.scale)[0]
        assert_attention_close(got[b], ref, bound, f"hca seq {b}")
    return got


def test_batch_invariant_decode_is_bitwise_across_batch_sizes():
    """With CSA_FLAG_BATCH_INVARIANT a sequence's selection and output bits do
    not depend on the batch it is decoded in: the first sequence decoded
    alone, in a batch of 8 and in a batch of 32 gives identical bytes (and the
    first 8 agree between 8 and 32); parity with the oracle holds as usual."""
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=32, n_ctx=16384, seed=15)
    B, H, d, HI, dI, m, W, k = w.batch, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = w.n_blocks
    p = K.params(m, W, k, H, d, HI, dI, w.scale, FMT[w.act], FMT[w.kv], FMT[w.idx],
                 flags=K.FLAG_BATCH_INVARIANT)
    vals = {n: draw_np(w, n) for n in ("q", "qI", "w", "kv", "kI", "window", "sinks")}
    kv_d, _ = both_stored(vals["kv"].reshape(-1, d), w.kv)
    kI_d, _ = both_stored(vals["kI"].reshape(-1, dI), w.idx)
    qI_d, _ = both_stored(vals["qI"].reshape(-1, dI), w.idx)
    rng = np.random.default_rng(15)
    q_pos = np.sort(rng.integers(3000, w.n_ctx + 1, size=B)).astype(np.int64)[::-1].copy()
    q_pos[0] = w.n_ctx
    q_d, win_d = act_dev(vals["q"], w.act), act_dev(vals["window"], w.act)
    w_d, pos_d, pos0_d, sinks_d = up(vals["w"]), up(q_pos), up(q_pos - W + 1), up(vals["sinks"])
    outs, sels = {}, {}
    for b in (1, 8, 32):
        sub = lambda st, per: K.Stored(st.fmt, st.data[:b * per], None if st.scales is None else st.scales[:b * per])
        out = torch.empty((b, H, d), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((b, k), dtype=torch.int32, device="cuda")
        ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, b, 1, nb), dtype=torch.uint8, device="cuda")
        K.csa_decode(p, b, q_d[:b], sub(qI_d, HI), w_d[:b], sub(kv_d, nb), sub(kI_d, nb), nb, win_d[:b], W,
                     pos0_d[:b], pos_d[:b], sinks_d, out, sel, ws)
        outs[b], sels[b] = down(out), down(sel)
    for b in (8, 32):
        assert np.array_equal(sels[b][:1], sels[1]) and np.array_equal(outs[b][:1], outs[1]), f"batch {b}"
    assert np.array_equal(sels[32][:8], sels[8]) and np.array_equal(outs[32][:8], outs[8])
    # parity of the invariant mode (first sequence)
    t = int(q_pos[0])
    kv_o, kI_o = orc_quantize(vals["kv"][0], w.kv), orc_quantize(vals["kI"][0], w.idx)
    scores = oracle.indexer(orc_quantize(vals["qI"][0].reshape(-1, dI), w.idx), vals["w"][0][None], kI_o, [t],
                            HI, m, W)[0]
    check_selection(sels[1][0], scores, min(oracle.n_elig(t, m, W), nb), k, what="seq 0")
    args = (act_orc(vals["q"][0], w.act), kv_o, sels[1][:1], act_orc(vals["window"][0], w.act), t - W + 1)
    ref = oracle.attention(*args, vals["sinks"], [t], H, m, W, w.scale)[0]
    bound = attention_bound_stored(*args, vals["sinks"], [t], H, m, W, w.scale)[0]
    got = synth.bf16_bits_to_f32_np(outs[1][0])
    assert_attention_close(got, ref, bound, "seq 0")
