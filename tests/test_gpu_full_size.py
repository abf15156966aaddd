"""Parity at the full sizes of the workloads, in the launch configuration the
benchmark times (the same entry points, shapes and arguments):

  * CSA decode, 32 sequences of 131,072 tokens: every sequence's selection and
    output checked against the oracle;
  * CSA prefill, bf16, T = 8192 (n_elig(t) > k for t > 2176, so the many-row
    top-k really selects): every 64th query row and the last one;
  * HCA decode, 8 sequences of 1,048,576 tokens pooled at m' = 128 on the
    device: two sequences (the first and the last) checked, pooling included.

Inputs come from the seeded generator.  Large tensors are drawn on the device
(synth.tensor_torch) and the rows the oracle needs are copied back, so both
sides read the same generated values; each side quantises them with its own
quantiser.  Checks of independent sequences / rows run in a thread pool (the
oracle's C calls release the interpreter lock).
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
from helpers import (FMT, assert_attention_close, attention_bound_stored, bf16_values_match,
                     check_selection, down, orc_quantize, quant_codes_match, up)
from synth.workloads import WORKLOADS, draw_np, draw_torch

pytestmark = pytest.mark.gpu


def _threads():
    return max(1, len(os.sched_getaffinity(0)))


def _pmap(fn, items):
    with ThreadPoolExecutor(_threads()) as ex:
        return list(ex.map(fn, items))


@pytest.fixture(autouse=True)
def _clean_status():
    K.csa_device_status(reset=True)
    yield
    assert K.csa_device_status(reset=True) == 0
    torch.cuda.empty_cache()


def _bf16_host(t):
    """bf16 device tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_csa_decode_full_size_every_sequence():
    w = WORKLOADS["csa_decode_128k_b32"]
    B, H, d, HI, dI, m, W, k = w.batch, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = w.n_blocks
    p = K.params(m, W, k, H, d, HI, dI, w.scale, FMT[w.act], FMT[w.kv], FMT[w.idx])
    kv = K.empty_stored(K.FP8_S64, B * nb, d)
    kI = K.empty_stored(K.MXFP4, B * nb, dI)
    host = {}
    for name, st, width in (("kv", kv, d), ("kI", kI, dI)):
        v = draw_torch(w, name)
        K.csa_quantize(v.reshape(-1, width), st)
        host[name] = down(v)          # the same generated values, for the oracle
        del v
    qI_v = draw_torch(w, "qI")
    qI = K.empty_stored(K.MXFP4, B * HI, dI)
    K.csa_quantize(qI_v.reshape(-1, dI), qI)
    q, wt, win, sinks = (draw_torch(w, n) for n in ("q", "w", "window", "sinks"))
    q_pos = torch.full((B,), w.n_ctx, dtype=torch.int64, device="cuda")
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, k, dtype=torch.int32, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, B, 1, nb), dtype=torch.uint8, device="cuda")
    K.csa_decode(p, B, q, qI, wt, kv, kI, nb, win, W, q_pos - W + 1, q_pos, sinks, out, sel, ws)
    torch.cuda.synchronize()
    got, got_sel = down(out.float()), down(sel)
    qh, qIh, wh, winh, sh = _bf16_host(q), down(qI_v), down(wt), _bf16_host(win), down(sinks)
    kv_h, kI_h = host["kv"], host["kI"]
    t = w.n_ctx

    def check(b):
        kv_o, kI_o = orc_quantize(kv_h[b], "fp8"), orc_quantize(kI_h[b], "mxfp4")
        qI_o = orc_quantize(qIh[b].reshape(-1, dI), "mxfp4")
        scores = oracle.indexer(qI_o, wh[b][None], kI_o, [t], HI, m, W)[0]
        check_selection(got_sel[b], scores, min(oracle.n_elig(t, m, W), nb), k, what=f"seq {b}")
        args = (oracle.Stored(oracle.BF16, qh[b]), kv_o, got_sel[b][None],
                oracle.Stored(oracle.BF16, winh[b]), t - W + 1)
        ref = oracle.attention(*args, sh, [t], H, m, W, w.scale)[0]
        bound = attention_bound_stored(*args, sh, [t], H, m, W, w.scale)[0]
        assert_attention_close(got[b], ref, bound, f"seq {b}")
        return b

    assert _pmap(check, range(B)) == list(range(B))


def test_csa_prefill_full_size_sampled_rows():
    w = WORKLOADS["csa_prefill_8k_bf16"]
    B, T, H, d, HI, dI, m, W, k = w.batch, w.n_ctx, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = T // m
    p = K.params(m, W, k, H, d, HI, dI, w.scale, K.BF16, K.BF16, K.BF16)
    t_ = {n: draw_torch(w, n) for n in ("x", "z", "bias", "q", "qI", "kI", "w", "sinks")}
    kv = K.empty_stored(K.BF16, B * nb, d)
    qI, kI = K.Stored(K.BF16, t_["qI"]), K.Stored(K.BF16, t_["kI"])
    out = torch.empty(B, T, H, d, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, T, k, dtype=torch.int32, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_PREFILL, B, T, nb), dtype=torch.uint8, device="cuda")
    K.csa_prefill(p, B, T, 0, t_["x"], T, 0, t_["z"], t_["bias"], t_["q"], qI, t_["w"], kv, kI, nb,
                  t_["sinks"], out, sel, ws)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, T, 64), [T - 1]]))
    assert (np.array([oracle.n_elig(int(t), m, W) for t in rows]) > k).sum() > 60
    got = down(out[:, rows].float())
    got_sel = down(sel[:, rows])
    x, z = _bf16_host(t_["x"]), _bf16_host(t_["z"])
    bias, wt, sinks = down(t_["bias"]), down(t_["w"]), down(t_["sinks"])
    q_rows = _bf16_host(t_["q"][:, rows])
    qI_rows = _bf16_host(t_["qI"][:, rows])
    kI_h = _bf16_host(t_["kI"])
    b = 0
    pooled = oracle.compress(oracle.Stored(oracle.BF16, x[b]), oracle.Stored(oracle.BF16, z[b]), bias, m)
    # the pooled entries the chunk wrote (bf16): both sides round their fp32
    # value once, so they may differ only on a rounding boundary
    assert bf16_values_match(_bf16_host(kv.data[:nb]), oracle.f32_to_bf16(pooled), pooled) == 0
    kv_o = oracle.Stored(oracle.BF16, oracle.f32_to_bf16(pooled))
    kI_o = oracle.Stored(oracle.BF16, kI_h[b])
    raw_o = oracle.Stored(oracle.BF16, x[b])
    groups = np.array_split(np.arange(len(rows)), _threads())

    def check(ix):
        if len(ix) == 0:
            return 0
        qIo = oracle.Stored(oracle.BF16, qI_rows[b][ix].reshape(-1, dI))
        scores = oracle.indexer(qIo, wt[b][rows[ix]], kI_o, rows[ix], HI, m, W)
        for a, i in enumerate(ix):
            t = int(rows[i])
            check_selection(got_sel[b, i], scores[a], min(oracle.n_elig(t, m, W), nb), k, what=f"t {t}")
        args = (oracle.Stored(oracle.BF16, q_rows[b][ix].reshape(-1, d)), kv_o, got_sel[b][ix], raw_o, 0)
        ref = oracle.attention(*args, sinks, rows[ix], H, m, W, w.scale)
        bound = attention_bound_stored(*args, sinks, rows[ix], H, m, W, w.scale)
        assert_attention_close(got[b][ix], ref, bound, f"rows {rows[ix][:3]}..")
        return len(ix)

    assert sum(_pmap(check, groups)) == len(rows)


def test_hca_decode_full_size_sampled_sequences():
    w = WORKLOADS["hca_decode_1m_b8"]
    B, N, H, d, m, W = w.batch, w.n_ctx, w.H, w.d, w.m, w.W
    nb = N // m
    p = K.params(m, W, 1, H, d, 1, 32, w.scale, FMT[w.act], FMT[w.kv], K.MXFP4)
    kv = K.empty_stored(K.FP8_S64, B * nb, d)
    bias = draw_torch(w, "bias")
    x, z = draw_torch(w, "x"), draw_torch(w, "z")
    K.csa_compress(p, d, x, z, bias, B * N, kv)
    win = torch.cat([x[:, N - W + 1:], draw_torch(w, "x_new")[:, None]], 1).contiguous()
    check_b = [0, B - 1]
    xs = {b: _bf16_host(x[b]) for b in check_b}
    zs = {b: _bf16_host(z[b]) for b in check_b}
    del x, z
    torch.cuda.empty_cache()
    q, sinks = draw_torch(w, "q"), draw_torch(w, "sinks")
    q_pos = torch.full((B,), N, dtype=torch.int64, device="cuda")
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(K.csa_workspace_size(p, K.OP_HCA_ATTN, B, 1, nb), dtype=torch.uint8, device="cuda")
    K.hca_attn(p, B, 1, q, kv, nb, win, W, q_pos - W + 1, q_pos, sinks, out, ws)
    torch.cuda.synchronize()
    got = down(out.float())
    kv_codes, kv_scales = down(kv.data), down(kv.scales)
    qh, winh, sh, bh = _bf16_host(q), _bf16_host(win), down(sinks), down(bias)

    def check(b):
        pooled = oracle.compress(oracle.Stored(oracle.BF16, xs[b]), oracle.Stored(oracle.BF16, zs[b]), bh, m)
        kv_o = orc_quantize(pooled, "fp8")
        rows = slice(b * nb, (b + 1) * nb)
        assert np.allclose(kv_scales[rows], kv_o.scales, rtol=1e-5, atol=0)
        assert quant_codes_match(kv_codes[rows], kv_o.data, pooled, np.repeat(kv_o.scales, 64, axis=1),
                                 "fp8") == 0
        args = (oracle.Stored(oracle.BF16, qh[b]), kv_o, None, oracle.Stored(oracle.BF16, winh[b]), N - W + 1)
        ref = oracle.attention(*args, sh, [N], H, m, W, w.scale)[0]
        bound = attention_bound_stored(*args, sh, [N], H, m, W, w.scale)[0]
        assert_attention_close(got[b], ref, bound, f"hca seq {b}")
        return b

    assert _pmap(check, check_b) == check_b
