"""Pins for the oracle's pooling, indexer, top-k and attention.

Every check compares the oracle with something independent of it: a hand-worked
example (golden fixtures), a closed form, an invariant, a library routine
(torch's scaled_dot_product_attention in float64, numpy sorting) or brute force
written from the definition on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines


def F32(orc, a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return orc.Stored(orc.F32, a.reshape(-1, a.shape[-1]))


# ------------------------------------------------------------------ pooling
def test_pooling_hand_example(orc):
    g = {ln[0]: ln[1:] for ln in golden_lines("pooling_hand.txt")}
    m = int(g["m"][0])
    x = np.array([float(v) for v in g["x"]], np.float32).reshape(-1, 1)
    z = np.zeros_like(x)
    b_log = np.log(np.arange(1, m + 1, dtype=np.float64)).astype(np.float32).reshape(m, 1)
    got = orc.compress(F32(orc, x), F32(orc, z), b_log, m)[:, 0]
    assert np.allclose(got, [float(v) for v in g["bias_log_r_plus_1"]], rtol=1e-6)
    got0 = orc.compress(F32(orc, x), F32(orc, z), np.zeros((m, 1), np.float32), m)[:, 0]
    assert np.allclose(got0, [float(v) for v in g["bias_zero"]], rtol=1e-7)


@pytest.mark.parametrize("m", [1, 4, 128])
def test_pooling_invariants(orc, m):
    rng = np.random.default_rng(m)
    d, nb = 8, 3
    z = rng.standard_normal((nb * m, d)).astype(np.float32)
    B = (0.1 * rng.standard_normal((m, d))).astype(np.float32)
    # gate weights sum to one: pooling a constant gives the constant back
    ones = np.full((nb * m, d), 1.75, np.float32)
    assert np.array_equal(orc.compress(F32(orc, ones), F32(orc, z), B, m),
                          np.full((nb, d), 1.75, np.float32))
    x = rng.standard_normal((nb * m, d)).astype(np.float32)
    # equal gate logits within a block -> plain mean of the block
    zc = np.repeat(rng.standard_normal((nb, 1, d)), m, axis=1).reshape(nb * m, d)
    got = orc.compress(F32(orc, x), F32(orc, zc.astype(np.float32)), np.zeros((m, d), np.float32), m)
    assert np.allclose(got, x.reshape(nb, m, d).astype(np.float64).mean(1), rtol=1e-6, atol=1e-7)
    # a gate that strongly prefers slot r picks out that token
    r = m - 1
    Bsel = np.zeros((m, d), np.float32)
    Bsel[r] = 80.0
    got = orc.compress(F32(orc, x), F32(orc, np.zeros_like(x)), Bsel, m)
    assert np.allclose(got, x.reshape(nb, m, d)[:, r], rtol=1e-6, atol=1e-30)
    # the weights are a per-channel softmax over slots: compare with torch
    zb = torch.from_numpy(z.reshape(nb, m, d)).double() + torch.from_numpy(B).double()
    ref = (torch.softmax(zb, dim=1) * torch.from_numpy(x.reshape(nb, m, d)).double()).sum(1)
    got = orc.compress(F32(orc, x), F32(orc, z), B, m)
    assert np.allclose(got, ref.numpy(), rtol=2e-7, atol=1e-7)


def test_pooling_reads_bf16_exactly(orc):
    import synth
    xb = synth.tensor_np(0, "pool_x", (8, 64), dtype="bf16")
    zb = synth.tensor_np(0, "pool_z", (8, 64), dtype="bf16")
    B = np.zeros((4, 64), np.float32)
    a = orc.compress(orc.Stored(orc.BF16, xb), orc.Stored(orc.BF16, zb), B, 4)
    b = orc.compress(F32(orc, synth.bf16_bits_to_f32_np(xb)),
                     F32(orc, synth.bf16_bits_to_f32_np(zb)), B, 4)
    assert np.array_equal(a, b)


# ------------------------------------------------------- indexer and top-k
def test_indexer_hand_example(orc):
    g = golden_lines("indexer_hand.txt")
    qI = F32(orc, [[1.0, 0.0]])
    kI = F32(orc, [[2.0, 0.0], [-1.0, 0.0]])
    t = 10  # m=1, W=0: both blocks eligible
    for (tag, s0, s1, _, top), w in zip(g, (1.0, -1.0)):
        s = orc.indexer(qI, np.array([[w]], np.float32), kI, [t], HI=1, m=1, W=0)[0]
        assert list(s) == [float(s0), float(s1)]
        sel = orc.topk(s[None, :], [t], 1, 1, 0)[0]
        assert list(sel) == [int(top)]


def test_n_elig_matches_definition(orc):
    # block j (tokens m*j .. m*j+m-1) is visible iff its last token < t - W
    for m, W in ((4, 64), (4, 0), (128, 128), (1, 3)):
        for t in range(0, 700, 7):
            brute = sum(1 for j in range(0, 800) if m * j + m - 1 < t - W)
            assert orc.n_elig(t, m, W) == brute


def test_indexer_special_cases(orc):
    rng = np.random.default_rng(5)
    HI, dI, nb = 3, 16, 40
    k = rng.standard_normal((nb, dI)).astype(np.float32)
    q = rng.standard_normal((HI, dI)).astype(np.float32)
    w = (0.1 * rng.standard_normal(HI)).astype(np.float32)
    t = 10_000
    s = orc.indexer(F32(orc, q), w[None], F32(orc, k), [t], HI=HI, m=4, W=0)[0]
    # one head, unit weight, all-positive vectors: the score is the dot product
    kp, qp = np.abs(k), np.abs(q[:1])
    s1 = orc.indexer(F32(orc, qp), np.ones((1, 1), np.float32), F32(orc, kp), [t], 1, 4, 0)[0]
    assert np.allclose(s1, kp.astype(np.float64) @ qp[0].astype(np.float64), rtol=1e-6)
    # heads whose dot product is negative contribute nothing (ReLU)
    dots = k.astype(np.float64) @ q.T.astype(np.float64)
    for j in range(nb):
        keep = dots[j] > 0
        qq = q[keep]
        if keep.sum() == 0:
            assert s[j] == 0
            continue
        sj = orc.indexer(F32(orc, qq), w[keep][None], F32(orc, k[j:j + 1]), [t], int(keep.sum()), 4, 0)
        assert np.isclose(sj[0, 0], s[j], rtol=1e-6)
    # a head with weight zero is ignored; negating every weight negates the score
    s_neg = orc.indexer(F32(orc, q), -w[None], F32(orc, k), [t], HI, 4, 0)[0]
    assert np.array_equal(s_neg, -s)
    # scores exist only for eligible blocks
    t2 = 4 * 10 + 7
    s2 = orc.indexer(F32(orc, q), w[None], F32(orc, k), [t2], HI, 4, 7)[0]
    assert np.all(np.isfinite(s2[:10])) and np.all(s2[10:] == -np.inf)


def test_topk_against_sorting(orc):
    rng = np.random.default_rng(2)
    rows, n, k = 30, 50, 8
    s = rng.standard_normal((rows, n)).astype(np.float32)
    s[3] = 0.0                          # all ties -> lowest indices
    s[4, :20] = 1.0                     # ties at the threshold
    s[4, 20:] = -1.0
    s[5] = np.round(s[5])               # many ties
    q_pos = np.full(rows, 10_000)
    q_pos[6] = 4 * 5                    # n_elig = 5 < k -> padding
    q_pos[7] = 0                        # nothing eligible
    idx = orc.topk(s, q_pos, k, 4, 0)
    for r in range(rows):
        ne = min(orc.n_elig(int(q_pos[r]), 4, 0), n)
        order = np.lexsort((np.arange(ne), -s[r, :ne].astype(np.float64)))
        want = np.sort(order[:min(k, ne)])
        got = idx[r]
        assert list(got[:len(want)]) == list(want)
        assert np.all(got[len(want):] == -1)
    assert list(idx[3]) == list(range(k))
    assert list(idx[4]) == list(range(k))
    assert list(idx[6]) == [0, 1, 2, 3, 4, -1, -1, -1]
    assert np.all(idx[7] == -1)


# ----------------------------------------------------------------- attention
def test_attention_hand_example(orc):
    g = {ln[0]: float(ln[1]) for ln in golden_lines("attention_hand.txt")}
    c = F32(orc, [[3.0], [7.0]])
    q = F32(orc, [[1.0]])
    raw = F32(orc, np.zeros((9, 1)))
    sel = np.array([[0, 1]], np.int32)
    for sink, key in ((-np.inf, "no_sink"), (0.0, "sink_zero")):
        o = orc.attention(q, c, sel, raw, 0, np.array([sink], np.float32), [8], H=1, m=4, W=0,
                          scale=1.0)
        assert abs(o[0, 0, 0] - g[key]) < 1e-9
    o = orc.attention(q, c, sel, raw, 0, None, [8], H=1, m=4, W=0, scale=1.0)
    assert abs(o[0, 0, 0] - g["no_sink"]) < 1e-9
    # HCA (dense over every eligible block) gives the same on this input
    o = orc.attention(q, c, None, raw, 0, None, [8], H=1, m=4, W=0, scale=1.0)
    assert abs(o[0, 0, 0] - g["no_sink"]) < 1e-9


def _sdpa_ref(qh, keys, sinks, scale):
    """torch SDPA in float64 with the sink as an extra key of value 0 whose
    logit is set by the additive mask."""
    H, d = qh.shape
    n = keys.shape[0]
    q = torch.from_numpy(qh).double()[None, :, None, :]                # [1,H,1,d]
    kk = torch.cat([torch.from_numpy(keys).double(), torch.zeros(1, d, dtype=torch.float64)])
    k = kk[None, None].expand(1, H, n + 1, d)
    mask = torch.zeros(1, H, 1, n + 1, dtype=torch.float64)
    if sinks is None:
        mask[..., n] = -math.inf
    else:
        mask[0, :, 0, n] = torch.from_numpy(sinks.astype(np.float64))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, k, attn_mask=mask, scale=scale)
    return o[0, :, 0, :].numpy()


@pytest.mark.parametrize("t,W,k", [(200, 16, 100), (200, 16, 5), (45, 0, 3), (10, 16, 4), (0, 16, 4)])
def test_attention_against_sdpa(orc, t, W, k):
    """CSA output equals SDPA over the set the definition names: the selected
    pooled entries plus raw tokens t-W < i <= t, with the sink."""
    rng = np.random.default_rng(t + W + k)
    H, d, m = 4, 16, 4
    nb = 60
    kv = rng.standard_normal((nb, d)).astype(np.float32)
    raw = rng.standard_normal((t + 1, d)).astype(np.float32)
    q = rng.standard_normal((H, d)).astype(np.float32)
    sinks = rng.standard_normal(H).astype(np.float32)
    ne = min(max(0, (t - W) // m), nb)
    chosen = np.sort(rng.permutation(ne)[:min(k, ne)]).astype(np.int32)
    sel = np.full((1, k), -1, np.int32)
    sel[0, :len(chosen)] = chosen
    scale = 1 / math.sqrt(d)
    o = orc.attention(F32(orc, q), F32(orc, kv), sel, F32(orc, raw), 0, sinks, [t], H, m, W,
                      scale)[0]
    window = [i for i in range(0, t + 1) if t - W < i <= t]
    keys = np.concatenate([kv[chosen], raw[window]]).astype(np.float64)
    ref = _sdpa_ref(q.astype(np.float64), keys, sinks, scale)
    assert np.allclose(o, ref, rtol=1e-10, atol=1e-12)


def test_topk_all_and_no_window_is_dense_attention(orc):
    """With k >= n_elig and W = 0, CSA reduces to dense attention over every
    eligible pooled entry (and equals HCA at the same m)."""
    rng = np.random.default_rng(9)
    H, d, m, nb, t = 2, 8, 4, 30, 100
    HI, dI = 2, 8
    kv = rng.standard_normal((nb, d)).astype(np.float32)
    q = rng.standard_normal((H, d)).astype(np.float32)
    qI = rng.standard_normal((HI, dI)).astype(np.float32)
    kI = rng.standard_normal((nb, dI)).astype(np.float32)
    w = rng.standard_normal((1, HI)).astype(np.float32)
    raw = rng.standard_normal((t + 1, d)).astype(np.float32)
    sinks = rng.standard_normal(H).astype(np.float32)
    sel, o = orc.csa(F32(orc, q), F32(orc, kv), F32(orc, qI), w, F32(orc, kI), F32(orc, raw), 0,
                     sinks, [t], H, HI, m, 0, 32, 0.3)
    ne = t // m
    assert list(sel[0, :ne]) == list(range(ne)) and np.all(sel[0, ne:] == -1)
    o_hca = orc.attention(F32(orc, q), F32(orc, kv), None, F32(orc, raw), 0, sinks, [t], H, m, 0, 0.3)
    assert np.allclose(o, o_hca, rtol=1e-12, atol=1e-14)
    ref = _sdpa_ref(q.astype(np.float64), kv[:ne].astype(np.float64), sinks, 0.3)
    assert np.allclose(o[0], ref, rtol=1e-10, atol=1e-12)


def test_sink_limits_and_single_item(orc):
    d = 4
    v = F32(orc, [[1.0, -2.0, 3.0, 0.5]])
    q = F32(orc, [[0.3, 0.1, -0.2, 0.9]])
    raw = F32(orc, np.zeros((1, d)))
    sel = np.array([[0]], np.int32)
    t = 8  # m=4, W=0 -> blocks 0,1 eligible; only block 0 is given
    o = orc.attention(q, v, sel, raw, 0, None, [t], 1, 4, 0, 1.0)[0, 0]
    assert np.allclose(o, [1.0, -2.0, 3.0, 0.5])           # one item, no sink: o = v
    o = orc.attention(q, v, sel, raw, 0, np.array([60.0], np.float32), [t], 1, 4, 0, 1.0)[0, 0]
    assert np.all(np.abs(o) < 1e-20)                        # sink dominates: o -> 0
    o = orc.attention(q, v, sel, raw, 0, np.array([-1e30], np.float32), [t], 1, 4, 0, 1.0)[0, 0]
    assert np.allclose(o, [1.0, -2.0, 3.0, 0.5])


def test_csa_is_causal(orc):
    """Changing raw tokens after t, or pooled blocks that are not eligible,
    leaves the output at t unchanged."""
    rng = np.random.default_rng(11)
    H, d, m, W, t, nb = 2, 8, 4, 8, 50, 20
    HI, dI = 2, 8
    kv = rng.standard_normal((nb, d)).astype(np.float32)
    q = rng.standard_normal((H, d)).astype(np.float32)
    qI = rng.standard_normal((HI, dI)).astype(np.float32)
    kI = rng.standard_normal((nb, dI)).astype(np.float32)
    w = rng.standard_normal((1, HI)).astype(np.float32)
    raw = rng.standard_normal((nb * m, d)).astype(np.float32)
    sinks = np.zeros(H, np.float32)
    args = dict(H=H, HI=HI, m=m, W=W, k=3, scale=0.5)
    sel, o = orc.csa(F32(orc, q), F32(orc, kv), F32(orc, qI), w, F32(orc, kI), F32(orc, raw), 0,
                     sinks, [t], **args)
    ne = (t - W) // m
    raw2, kv2, kI2 = raw.copy(), kv.copy(), kI.copy()
    raw2[t + 1:] = 99.0
    kv2[ne:] = -99.0
    kI2[ne:] = 50.0
    sel2, o2 = orc.csa(F32(orc, q), F32(orc, kv2), F32(orc, qI), w, F32(orc, kI2), F32(orc, raw2),
                       0, sinks, [t], **args)
    assert np.array_equal(sel, sel2) and np.array_equal(o, o2)
    raw3 = raw.copy()
    raw3[t] += 1.0                                           # the query's own token is attended
    _, o3 = orc.csa(F32(orc, q), F32(orc, kv), F32(orc, qI), w, F32(orc, kI), F32(orc, raw3), 0,
                    sinks, [t], **args)
    assert not np.array_equal(o, o3)


def test_csa_composes_its_steps(orc):
    """The whole-step routine equals indexer -> top-k -> attention run one by one,
    with raw rows supplied as a window buffer (decode layout)."""
    import synth
    H, d, HI, dI, m, W, k = 4, 64, 2, 32, 4, 16, 6
    nb, t = 40, 160
    s = 7
    q = orc.Stored(orc.BF16, synth.tensor_np(s, "q", (H, d), dtype="bf16"))
    kv = orc.quantize_fp8_s64(synth.tensor_np(s, "kv", (nb, d)))
    qI = orc.quantize_mxfp4(synth.tensor_np(s, "qI", (HI, dI)))
    kI = orc.quantize_mxfp4(synth.tensor_np(s, "kI", (nb, dI)))
    w = synth.tensor_np(s, "w", (1, HI), std=0.1)
    win = orc.Stored(orc.BF16, synth.tensor_np(s, "win", (W, d), dtype="bf16"))
    sinks = synth.tensor_np(s, "sink", (H,))
    pos0 = t - W + 1
    sel, o = orc.csa(q, kv, qI, w, kI, win, pos0, sinks, [t], H, HI, m, W, k, 0.125)
    sc = orc.indexer(qI, w, kI, [t], HI, m, W)
    sel2 = orc.topk(sc, [t], k, m, W)
    o2 = orc.attention(q, kv, sel2, win, pos0, sinks, [t], H, m, W, 0.125)
    assert np.array_equal(sel, sel2) and np.array_equal(o, o2)


@pytest.mark.parametrize("t,W,raw_pos0", [(50, 16, 0), (50, 16, 40), (5, 16, 0), (0, 1, 0), (30, 64, 10)])
def test_window_only_attention_against_sdpa(orc, t, W, raw_pos0):
    """The MTP block's window-only attention (no pooled entry) is SDPA over the
    raw tokens t-W < i <= t that the raw buffer holds, with the sink: the
    oracle's attention with an empty entry table must equal it."""
    rng = np.random.default_rng(100 + t + W + raw_pos0)
    H, d, m = 3, 16, 4
    raw = rng.standard_normal((t + 1 - raw_pos0, d)).astype(np.float32)
    q = rng.standard_normal((H, d)).astype(np.float32)
    sinks = rng.standard_normal(H).astype(np.float32)
    scale = 1 / math.sqrt(d)
    empty = F32(orc, np.zeros((0, d), np.float32))
    o = orc.attention(F32(orc, q), empty, None, F32(orc, raw), raw_pos0, sinks, [t], H, m, W, scale)[0]
    window = [i for i in range(raw_pos0, t + 1) if t - W < i <= t]
    keys = raw[[i - raw_pos0 for i in window]].astype(np.float64)
    ref = _sdpa_ref(q.astype(np.float64), keys, sinks, scale)
    assert np.allclose(o, ref, rtol=1e-10, atol=1e-12)
