"""The interleaved CSA / HCA stack with incremental pooling (row a7): a prefill
chunk right after a prior cache, then decode steps, on four layers (CSA, HCA,
CSA, HCA) through compressed_sparse_attention_13_b200.stack.  Checked against
the oracle:
  * entries pooled during the chunk and the decode steps equal the oracle's
    pooling of the same tokens, quantised by its own quantiser (codes may
    differ only on a rounding boundary);
  * every decode output and a sample of chunk outputs equal the oracle's
    attention over the stored caches (the GPU's stored bytes, as the
    matching rule asks), with CSA selections validated against the oracle's
    indexer scores.
Reduced sizes: a 2048-token prior cache, a 256-token chunk, 32 decode steps,
k = 128; the kernels' full shapes (64 heads x 512, 64 indexer heads x 128)."""
import math

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from compressed_sparse_attention_13_b200.stack import Layer, LayerSpec
from helpers import (assert_close_abs, both_stored, check_selection, down, orc_quantize,
                     quant_codes_match, up)

pytestmark = pytest.mark.gpu

H, D, HI, DI, W = 64, 512, 64, 128, 128
PRIOR, CHUNK, STEPS, TOPK = 2048, 256, 32, 128
SCALE = 1 / math.sqrt(D)


def _val(bits):
    """fp32 values of bf16 bit patterns (exact)."""
    return synth.bf16_bits_to_f32_np(bits)


def _run_layer(kind, seed):
    m = 4 if kind == "csa" else 128
    p = K.params(m, W, TOPK if kind == "csa" else 1, H, D, HI, DI, SCALE, K.BF16, K.FP8_S64, K.MXFP4)
    spec = LayerSpec(kind, p, PRIOR, CHUNK + STEPS)
    L = Layer(spec)
    n_new = CHUNK + STEPS
    g = lambda name, shape, std=1.0, dt="f32": synth.tensor_np(seed, f"stack/{kind}/{name}", shape, std, dt)
    prior_kv = g("prior_kv", (PRIOR // m, D))
    xb_prior = g("x_prior", (W - 1, D), dt="bf16")     # bf16 bit patterns
    xb, zb = g("x", (n_new, D), dt="bf16"), g("z", (n_new, D), dt="bf16")
    bias = g("bias", (m, D), 0.1)
    qb = g("q", (n_new, H, D), dt="bf16")
    sinks = g("sinks", (H,))
    x_prior, x, z, q = _val(xb_prior), _val(xb), _val(zb), _val(qb)
    kv_prior_d, _ = both_stored(prior_kv, "fp8")
    L.kv.data[:PRIOR // m].copy_(kv_prior_d.data)
    L.kv.scales[:PRIOR // m].copy_(kv_prior_d.scales)
    L.set_prior_window(up(xb_prior, True))
    inp = dict(x=x, z=z, bias=bias, q=q, sinks=sinks, x_prior=x_prior, m=m, p=p)
    if kind == "csa":
        prior_kI = g("prior_kI", (PRIOR // m, DI))
        xIb, zIb = g("xI", (n_new, DI), dt="bf16"), g("zI", (n_new, DI), dt="bf16")
        xI, zI = _val(xIb), _val(zIb)
        biasI = g("biasI", (m, DI), 0.1)
        qI = g("qI", (n_new, HI, DI))
        w = g("w", (n_new, HI), 0.1)
        kI_prior_d, _ = both_stored(prior_kI, "mxfp4")
        L.kI.data[:PRIOR // m].copy_(kI_prior_d.data)
        L.kI.scales[:PRIOR // m].copy_(kI_prior_d.scales)
        qI_d, _ = both_stored(qI.reshape(-1, DI), "mxfp4")
        inp.update(xI=xI, zI=zI, biasI=biasI, qI=qI, w=w, xIb=xIb, zIb=zIb)
    bias_d = up(bias)
    biasI_d = up(inp["biasI"]) if kind == "csa" else None
    q_d = up(qb, True)
    # prefill chunk
    L.append(up(xb[:CHUNK], True), up(zb[:CHUNK], True),
             up(inp["xIb"][:CHUNK], True) if kind == "csa" else None,
             up(inp["zIb"][:CHUNK], True) if kind == "csa" else None)
    out_chunk = torch.empty((CHUNK, H, D), dtype=torch.bfloat16, device="cuda")
    sel_chunk = torch.empty((CHUNK, TOPK), dtype=torch.int32, device="cuda")
    if kind == "csa":
        qIc = K.Stored(K.MXFP4, qI_d.data[:CHUNK * HI], qI_d.scales[:CHUNK * HI])
        L.prefill(CHUNK, q_d[:CHUNK], qIc, up(inp["w"][:CHUNK]), up(sinks), out_chunk, sel_chunk,
                  bias_d, biasI_d)
    else:
        L.prefill(CHUNK, q_d[:CHUNK], None, None, up(sinks), out_chunk, None, bias_d)
    # decode steps
    out_dec = torch.empty((STEPS, H, D), dtype=torch.bfloat16, device="cuda")
    sel_dec = torch.empty((STEPS, TOPK), dtype=torch.int32, device="cuda")
    for s in range(STEPS):
        i = CHUNK + s
        L.append(up(xb[i:i + 1], True), up(zb[i:i + 1], True),
                 up(inp["xIb"][i:i + 1], True) if kind == "csa" else None,
                 up(inp["zIb"][i:i + 1], True) if kind == "csa" else None)
        if kind == "csa":
            qIs = K.Stored(K.MXFP4, qI_d.data[i * HI:(i + 1) * HI], qI_d.scales[i * HI:(i + 1) * HI])
            L.decode(q_d[i], qIs, up(inp["w"][i]), up(sinks), out_dec[s], sel_dec[s], bias_d, biasI_d)
        else:
            L.decode(q_d[i], None, None, up(sinks), out_dec[s], None, bias_d)
    torch.cuda.synchronize()
    assert K.csa_device_status(reset=True) == 0
    res = dict(out_chunk=down(out_chunk.float()), sel_chunk=down(sel_chunk), out_dec=down(out_dec.float()),
               sel_dec=down(sel_dec), kv=K.Stored(K.FP8_S64, down(L.kv.data), down(L.kv.scales)),
               pooled=L._pooled)
    if kind == "csa":
        res["kI"] = K.Stored(K.MXFP4, down(L.kI.data), down(L.kI.scales))
    return inp, res


def _check_layer(kind, inp, res):
    m, p = inp["m"], inp["p"]
    n_new = CHUNK + STEPS
    first, last = PRIOR // m, res["pooled"]
    # pooled entries vs the oracle's own pooling + quantisation
    xs = oracle.Stored(oracle.F32, inp["x"][: (last - first) * m])
    zs = oracle.Stored(oracle.F32, inp["z"][: (last - first) * m])
    pre = oracle.compress(xs, zs, inp["bias"], m)
    o = orc_quantize(pre, "fp8")
    got_codes = res["kv"].data[first:last]
    assert np.allclose(res["kv"].scales[first:last], o.scales, rtol=1e-5, atol=0)
    assert quant_codes_match(got_codes, o.data, pre, np.repeat(o.scales, 64, axis=1), "fp8") == 0
    if kind == "csa":
        preI = oracle.compress(oracle.Stored(oracle.F32, inp["xI"][: (last - first) * m]),
                               oracle.Stored(oracle.F32, inp["zI"][: (last - first) * m]),
                               inp["biasI"], m)
        oI = orc_quantize(preI, "mxfp4")
        assert np.array_equal(res["kI"].scales[first:last], oI.scales)
    # attention against the oracle over the stored caches
    kv_o = oracle.Stored(oracle.FP8_S64, res["kv"].data, res["kv"].scales)
    raw = oracle.Stored(oracle.F32, np.concatenate([inp["x_prior"], inp["x"]]).astype(np.float32))
    raw_pos0 = PRIOR - (W - 1)
    q_all = oracle.Stored(oracle.F32, inp["q"].reshape(-1, D))
    rows = list(range(0, CHUNK, 37)) + [CHUNK - 1] + [CHUNK + s for s in range(STEPS)]
    for i in rows:
        t = PRIOR + i
        got = res["out_chunk"][i] if i < CHUNK else res["out_dec"][i - CHUNK]
        qi = oracle.Stored(oracle.F32, inp["q"][i].reshape(-1, D))
        if kind == "csa":
            kI_o = oracle.Stored(oracle.MXFP4, res["kI"].data, res["kI"].scales)
            qIi = orc_quantize(inp["qI"][i], "mxfp4")
            scores = oracle.indexer(qIi, inp["w"][i][None], kI_o, [t], HI, m, W)[0]
            ne = min(oracle.n_elig(t, m, W), res["kv"].data.shape[0])
            sel = res["sel_chunk"][i] if i < CHUNK else res["sel_dec"][i - CHUNK]
            check_selection(sel, scores, ne, TOPK, what=f"{kind} token {t}")
            ref = oracle.attention(qi, kv_o, sel[None], raw, raw_pos0, inp["sinks"], [t], H, m, W, SCALE)[0]
        else:
            ref = oracle.attention(qi, kv_o, None, raw, raw_pos0, inp["sinks"], [t], H, m, W, SCALE)[0]
        assert_close_abs(got, ref, 2e-2, f"{kind} token {t}")


def test_interleaved_stack_with_incremental_pooling():
    K.csa_device_status(reset=True)
    for li, kind in enumerate(["csa", "hca", "csa", "hca"]):
        inp, res = _run_layer(kind, seed=40 + li)
        _check_layer(kind, inp, res)
