"""The interleaved CSA / HCA stack with incremental pooling (row a7): a prefill
chunk right after a prior cache, then decode steps, on four layers (CSA, HCA,
CSA, HCA) through compressed_sparse_attention_13_b200.stack.  Checked against
the oracle:
  * entries pooled during the chunk and the decode steps (FP8 entries, and the
    MXFP4 indexer keys of CSA layers: scales and codes) equal the oracle's
    pooling of the same tokens, quantised by its own quantiser (codes may
    differ only on a rounding boundary);
  * every checked output equals the oracle's attention over caches the oracle
    builds itself (its own quantisation of the prior values, its own pooling
    of the new tokens), with CSA selections validated against the oracle's
    indexer scores; bf16 outputs meet the 2e-2 rule and the derived bound.
Reduced sizes: a 2048-token prior cache, k = 128, the kernels' full shapes
(64 heads x 512, 64 indexer heads x 128); chunks aligned to both m and m'
(256 tokens) and unaligned (254 for CSA, 200 for HCA: the partial block is
pooled later by the decode step that completes it).  The full-size stack
(1M context, 4096-token chunk, 256 decode steps, k = 1024) is checked on
sampled rows."""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from compressed_sparse_attention_13_b200.stack import Layer, LayerSpec
from helpers import (assert_attention_close, attention_bound_stored, both_stored, check_selection,
                     down, orc_quantize, quant_codes_match, up)

pytestmark = pytest.mark.gpu

H, D, HI, DI, W = 64, 512, 64, 128, 128
SCALE = 1 / math.sqrt(D)


def _threads():
    return max(1, len(os.sched_getaffinity(0)))


def _unpack(a):
    a = np.asarray(a).astype(np.uint8)
    return np.stack([a & 15, a >> 4], -1).reshape(a.shape[0], -1)


def _bf16_host(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class _Draw:
    """Inputs of one layer: drawn on the device from the seeded generator
    (stream names `{prefix}/{name}`), copied back to the host on demand."""

    def __init__(self, prefix, seed):
        self.prefix, self.seed, self.dev = prefix, seed, {}

    def __call__(self, name, shape, std=1.0, dt="f32"):
        if name not in self.dev:
            self.dev[name] = synth.tensor_torch(self.seed, f"{self.prefix}/{name}", shape, std, dt)
        return self.dev[name]

    def host(self, name):
        t = self.dev[name]
        return _bf16_host(t) if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def _run_layer(kind, g, prior, chunk, steps, topk, win=W):
    """Run one layer (prior cache, chunk, decode steps) on the device; returns
    the outputs and selections of the chunk and of the decode steps, and the
    layer's caches."""
    m = 128 if kind == "hca" else 4
    p = K.params(m, win, topk if kind == "csa" else 1, H, D, HI, DI, SCALE, K.BF16, K.FP8_S64, K.MXFP4)
    n_new = chunk + steps
    L = Layer(LayerSpec(kind, p, prior, n_new))
    if kind != "window":
        K.csa_quantize(g("prior_kv", (prior // m, D)), K.Stored(K.FP8_S64, L.kv.data[:prior // m],
                                                                L.kv.scales[:prior // m]))
    if win > 1:
        L.set_prior_window(g("x_prior", (win - 1, D), dt="bf16"))
    x, z = g("x", (n_new, D), dt="bf16"), g("z", (n_new, D), dt="bf16")
    bias, q, sinks = g("bias", (m, D), 0.1), g("q", (n_new, H, D), dt="bf16"), g("sinks", (H,))
    out = torch.empty(n_new, H, D, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(n_new, topk, dtype=torch.int32, device="cuda")
    csa = kind == "csa"
    if csa:
        K.csa_quantize(g("prior_kI", (prior // m, DI)), K.Stored(K.MXFP4, L.kI.data[:prior // m],
                                                                 L.kI.scales[:prior // m]))
        xI, zI = g("xI", (n_new, DI), dt="bf16"), g("zI", (n_new, DI), dt="bf16")
        biasI, wt = g("biasI", (m, DI), 0.1), g("w", (n_new, HI), 0.1)
        qI = K.empty_stored(K.MXFP4, n_new * HI, DI)
        K.csa_quantize(g("qI", (n_new * HI, DI)), qI)
    rows = lambda st, a, b: K.Stored(st.fmt, st.data[a:b], st.scales[a:b])
    L.append(x[:chunk], z[:chunk], xI[:chunk] if csa else None, zI[:chunk] if csa else None)
    L.prefill(chunk, q[:chunk], rows(qI, 0, chunk * HI) if csa else None, wt[:chunk] if csa else None,
              sinks, out[:chunk], sel[:chunk] if csa else None, bias, biasI if csa else None)
    for s in range(steps):
        i = chunk + s
        L.append(x[i:i + 1], z[i:i + 1], xI[i:i + 1] if csa else None, zI[i:i + 1] if csa else None)
        L.decode(q[i], rows(qI, i * HI, (i + 1) * HI) if csa else None, wt[i] if csa else None, sinks,
                 out[i], sel[i] if csa else None, bias, biasI if csa else None)
    torch.cuda.synchronize()
    assert K.csa_device_status(reset=True) == 0
    res = dict(out=out, sel=sel, m=m, pooled=L._pooled,
               kv=None if L.kv is None else K.Stored(K.FP8_S64, down(L.kv.data), down(L.kv.scales)))
    if csa:
        res["kI"] = K.Stored(K.MXFP4, down(L.kI.data), down(L.kI.scales))
    return res


def _oracle_caches(kind, g, res, prior, n_pooled_new):
    """The oracle's own caches: its quantisation of the prior values and its
    pooling + quantisation of the new tokens' complete blocks.  Also checks
    the library's pooled rows against them."""
    m = res["m"]
    if kind == "window":   # the MTP block keeps no pooled cache
        return dict(kv=oracle.Stored(oracle.FP8_S64, np.zeros((0, D), np.uint8), np.zeros((0, D // 64), np.float32)))
    first, last = prior // m, res["pooled"]
    assert last - first == n_pooled_new
    x, z = g.host("x"), g.host("z")
    pre = oracle.compress(oracle.Stored(oracle.BF16, x[: (last - first) * m]),
                          oracle.Stored(oracle.BF16, z[: (last - first) * m]), g.host("bias"), m)
    o = orc_quantize(pre, "fp8")
    assert np.allclose(res["kv"].scales[first:last], o.scales, rtol=1e-5, atol=0)
    assert quant_codes_match(res["kv"].data[first:last], o.data, pre, np.repeat(o.scales, 64, axis=1),
                             "fp8") == 0
    prior_o = orc_quantize(g.host("prior_kv"), "fp8")
    kv_o = oracle.Stored(oracle.FP8_S64, np.concatenate([prior_o.data, o.data]),
                         np.concatenate([prior_o.scales, o.scales]))
    caches = dict(kv=kv_o)
    if kind == "csa":
        preI = oracle.compress(oracle.Stored(oracle.BF16, g.host("xI")[: (last - first) * m]),
                               oracle.Stored(oracle.BF16, g.host("zI")[: (last - first) * m]),
                               g.host("biasI"), m)
        oI = orc_quantize(preI, "mxfp4")
        got = res["kI"]
        assert np.array_equal(got.scales[first:last], oI.scales)
        per_el = np.repeat(2.0 ** (oI.scales.astype(np.float64) - 127), 32, axis=1)
        assert quant_codes_match(_unpack(got.data[first:last]), _unpack(oI.data), preI, per_el,
                                 "mxfp4") == 0
        priorI = orc_quantize(g.host("prior_kI"), "mxfp4")
        caches["kI"] = oracle.Stored(oracle.MXFP4, np.concatenate([priorI.data, oI.data]),
                                     np.concatenate([priorI.scales, oI.scales]), DI)
    return caches


def _check_rows(kind, g, res, caches, prior, check_rows, topk, win=W):
    """Outputs (and CSA selections) of the given new-token rows against the oracle."""
    m = res["m"]
    W = win  # noqa: N806 (the window of this layer)
    raw = oracle.Stored(oracle.BF16, np.concatenate([g.host("x_prior"), g.host("x")]) if W > 1 else g.host("x"))
    raw_pos0 = prior - (W - 1) if W > 0 else prior
    q = g.host("q")
    sinks = g.host("sinks")
    rows = np.asarray(check_rows, np.int64)
    ri = torch.as_tensor(rows, device=res["out"].device)
    got = down(res["out"][ri].float())
    sel = down(res["sel"][ri])
    qI_all = g.host("qI").reshape(-1, HI, DI) if kind == "csa" else None
    n_ent = caches["kv"].rows

    def one(a):
        i = int(rows[a])
        t = prior + i
        s = None
        if kind == "csa":
            qIi = orc_quantize(qI_all[i], "mxfp4")
            scores = oracle.indexer(qIi, g.host("w")[i][None], caches["kI"], [t], HI, m, W)[0]
            ne = min(oracle.n_elig(t, m, W), n_ent)
            check_selection(sel[a], scores, ne, topk, what=f"{kind} token {t}")
            s = sel[a][None]
        args = (oracle.Stored(oracle.BF16, q[i].reshape(-1, D)), caches["kv"], s, raw, raw_pos0)
        ref = oracle.attention(*args, sinks, [t], H, m, W, SCALE)[0]
        bound = attention_bound_stored(*args, sinks, [t], H, m, W, SCALE)[0]
        assert_attention_close(got[a], ref, bound, f"{kind} token {t}")
        return i

    with ThreadPoolExecutor(_threads()) as ex:
        assert list(ex.map(one, range(len(rows)))) == list(rows)


@pytest.mark.parametrize("chunks", [(256, 256, 32), (254, 200, 64)],
                         ids=["aligned_chunk", "unaligned_chunk"])
def test_interleaved_stack_with_incremental_pooling(chunks):
    prior, topk = 2048, 128
    csa_chunk, hca_chunk, steps = chunks
    K.csa_device_status(reset=True)
    # four layers CSA, HCA, CSA, HCA and the MTP block (window only)
    for li, kind in enumerate(["csa", "hca", "csa", "hca", "window"]):
        chunk = hca_chunk if kind == "hca" else csa_chunk
        m = 128 if kind == "hca" else 4
        g = _Draw(f"stack/{kind}", 40 + li)
        res = _run_layer(kind, g, prior, chunk, steps, topk)
        caches = _oracle_caches(kind, g, res, prior, (chunk + steps) // m)
        rows = sorted(set(range(0, chunk, 37)) | {chunk - 1} | set(range(chunk, chunk + steps)))
        _check_rows(kind, g, res, caches, prior, rows, topk)


def test_interleaved_stack_full_size_sampled_rows():
    """The full four-layer stack of the benchmark (same seeded inputs): a prior
    cache of 1,044,480 tokens, a 4096-token chunk ending at 2^20, 256 decode
    steps, k = 1024.  Every pooled entry is checked; outputs on sampled rows:
    every 512th chunk query, the last one, and every 32nd decode step plus the
    last."""
    prior, chunk, steps, topk = 1_044_480, 4096, 256, 1024
    rows = sorted(set(range(0, chunk, 512)) | {chunk - 1} | set(range(chunk, chunk + steps, 32)) |
                  {chunk + steps - 1})
    K.csa_device_status(reset=True)
    for li, kind in enumerate(["csa", "hca", "csa", "hca"]):
        m = 4 if kind == "csa" else 128
        g = _Draw(f"stack_c4/{li}", 0)
        res = _run_layer(kind, g, prior, chunk, steps, topk)
        caches = _oracle_caches(kind, g, res, prior, (chunk + steps) // m)
        _check_rows(kind, g, res, caches, prior, rows, topk)
        del res, caches, g
        torch.cuda.empty_cache()


def test_csa_layer_without_window():
    """W = 0: no raw window at all; the prefill's raw buffer starts at the
    chunk (t0) and the decode steps attend to pooled entries only."""
    prior, topk, chunk, steps = 2048, 128, 256, 16
    K.csa_device_status(reset=True)
    g = _Draw("stack/nowin", 47)
    res = _run_layer("csa", g, prior, chunk, steps, topk, win=0)
    caches = _oracle_caches("csa", g, res, prior, (chunk + steps) // 4)
    rows = sorted(set(range(0, chunk, 41)) | {chunk - 1} | set(range(chunk, chunk + steps)))
    _check_rows("csa", g, res, caches, prior, rows, topk, win=0)
