"""The arithmetic-derived attention tolerance (helpers.attention_bound) checked
on the CPU, without the library:
  * it holds, with margin, for an emulation of the roundings the tensor-core
    attention performs (bf16 entries from FP8, bf16 P, fp32 sums, bf16 output);
  * it is tight enough that the mistakes it is meant to catch fail it: a
    dropped sink on sink-dominant rows, a window off by one, a dropped item on
    rows with few items.
The references are the oracle's attention on the oracle's stored inputs."""
import math

import numpy as np
import pytest

import oracle
import synth
from helpers import U_BF16, attention_bound, attention_items, orc_quantize, stored_values


def _bf16(x):
    """Round to the nearest bf16 (ties to even), as the kernel's conversions do."""
    b = synth.f32_to_bf16_bits_np(np.asarray(x, np.float32))
    return synth.bf16_bits_to_f32_np(b).astype(np.float64)


def _emulate(q, ent, ent_fp8, sel, raw, raw_pos0, sinks, q_pos, m, W, scale):
    """The kernel's arithmetic on the stored values: entries (if FP8) rounded
    to bf16, logits and sums in fp32, P rounded to bf16, output to bf16."""
    n_q, H, d = q.shape
    out = np.empty((n_q, H, d))
    for r in range(n_q):
        t = int(q_pos[r])
        ids, pos = attention_items(t, ent.shape[0], None if sel is None else sel[r], m, W,
                                   raw_pos0, raw.shape[0])
        Ke = _bf16(ent[ids]) if ent_fp8 else ent[ids]
        K = np.concatenate([Ke, raw[pos - raw_pos0]], 0).astype(np.float32)
        lg = (np.float32(scale) * (q[r].astype(np.float32) @ K.T)).astype(np.float32)
        M = np.maximum(lg.max(1), sinks.astype(np.float32))
        p = np.exp((lg - M[:, None]).astype(np.float32)).astype(np.float32)
        L = p.sum(1, dtype=np.float32) + np.exp(sinks.astype(np.float32) - M)
        Pb = _bf16(p).astype(np.float32)
        o = (Pb @ K) / L[:, None]
        out[r] = _bf16(o)
    return out


def _case(seed, n_ent, k, n_q, sink_shift=None, t_hi=None, q_pos=None):
    H, d, m, W = 64, 512, 4, 128
    scale = 1 / math.sqrt(d)
    q = synth.tensor_np(seed, "tm_q", (n_q, H, d), dtype="bf16")
    qv = synth.bf16_bits_to_f32_np(q).astype(np.float64)
    ent_o = orc_quantize(synth.tensor_np(seed, "tm_kv", (n_ent, d)), "fp8")
    ent = stored_values(ent_o)
    n_raw = W + 40
    rawb = synth.tensor_np(seed, "tm_raw", (n_raw, d), dtype="bf16")
    raw = synth.bf16_bits_to_f32_np(rawb).astype(np.float64)
    t_hi = m * n_ent + W + 20 if t_hi is None else t_hi
    rng = np.random.default_rng(seed)
    if q_pos is None:
        q_pos = rng.integers(0, t_hi + 1, size=n_q).astype(np.int64)
        q_pos[0] = t_hi
    q_pos = np.asarray(q_pos, np.int64)
    raw_pos0 = max(0, t_hi - n_raw + 1)
    sel = np.full((n_q, k), -1, np.int32)
    for i in range(n_q):
        ne = min(oracle.n_elig(int(q_pos[i]), m, W), n_ent)
        c = np.sort(rng.permutation(ne)[:min(k, ne)])
        sel[i, :len(c)] = c
    sinks = synth.tensor_np(seed, "tm_sink", (H,)).astype(np.float64)
    if sink_shift is not None:
        # sink logits above every attended logit: the sink dominates the denominator
        mx = np.full(H, -np.inf)
        for i in range(n_q):
            ids, pos = attention_items(int(q_pos[i]), n_ent, sel[i], m, W, raw_pos0, n_raw)
            K = np.concatenate([ent[ids], raw[pos - raw_pos0]], 0)
            if K.shape[0]:
                mx = np.maximum(mx, (scale * qv[i] @ K.T).max(1))
        sinks = mx + sink_shift
    stored = dict(q=oracle.Stored(oracle.BF16, q.reshape(-1, d)), kv=ent_o,
                  raw=oracle.Stored(oracle.BF16, rawb))
    return dict(qv=qv, ent=ent, raw=raw, sel=sel, q_pos=q_pos, raw_pos0=raw_pos0,
                sinks=sinks.astype(np.float32), H=H, d=d, m=m, W=W, scale=scale, stored=stored)


def _ref(c, sinks=None, W=None, sel=None):
    s = c["stored"]
    return oracle.attention(s["q"], s["kv"], c["sel"] if sel is None else sel, s["raw"], c["raw_pos0"],
                            c["sinks"] if sinks is None else sinks, c["q_pos"], c["H"], c["m"],
                            c["W"] if W is None else W, c["scale"])


def _bound(c):
    return attention_bound(c["qv"], c["ent"], True, c["sel"], c["raw"], c["raw_pos0"], c["sinks"],
                           c["q_pos"], c["m"], c["W"], c["scale"])


@pytest.mark.parametrize("sink_shift", [None, 2.0])
def test_bound_holds_for_the_kernel_arithmetic(sink_shift):
    c = _case(1, 700, 512, 4, sink_shift)
    ref, bound = _ref(c), _bound(c)
    emu = _emulate(c["qv"], c["ent"], True, c["sel"], c["raw"], c["raw_pos0"], c["sinks"],
                   c["q_pos"], c["m"], c["W"], c["scale"])
    ratio = np.abs(emu - ref) / bound
    assert ratio.max() < 0.6, ratio.max()
    # the derived bound is well inside the 2e-2 rule at these shapes (it is
    # looser only on heads whose softmax is dominated by a few items)
    assert np.median(bound) < 5e-3 and bound.max() < 2e-2, (np.median(bound), bound.max())


def test_bound_catches_a_dropped_sink_on_sink_dominant_rows():
    c = _case(2, 700, 512, 4, sink_shift=2.0)
    ref, bound = _ref(c), _bound(c)
    no_sink = _ref(c, sinks=np.full(c["H"], -np.inf, np.float32))
    diff = np.abs(no_sink - ref)
    # a kernel that ignored the sink would miss both rules on most elements
    assert (diff > bound).mean() > 0.9
    assert diff.max() > 2e-2


def test_bound_catches_window_mistakes_on_few_item_rows():
    W, m = 128, 4
    # positions below the window length: t + 1 raw tokens and no pooled entry;
    # a kernel that left out the query's own token is the oracle at t - 1
    few = np.array([0, 1, 2, 5, 9, 17], np.int64)
    c = _case(3, 3, 16, len(few), t_hi=150, q_pos=few)
    ref, bound = _ref(c), _bound(c)
    no_own = oracle.attention(c["stored"]["q"], c["stored"]["kv"], c["sel"], c["stored"]["raw"],
                              c["raw_pos0"], c["sinks"], few - 1, c["H"], m, W, c["scale"])
    diff = np.abs(no_own - ref)
    assert (diff > bound).any(axis=(1, 2))[1:].all(), "rows with t >= 1 must see their own token"
    assert diff.max() > 2e-2
    # at most three visible pooled blocks and a full window: the window start
    # off by one (W - 1) is caught on every row
    edge = W + np.array([0, 1, m, 2 * m + 1, 3 * m, 3 * m + 3], np.int64)
    c = _case(4, 3, 16, len(edge), t_hi=150, q_pos=edge)
    ref, bound = _ref(c), _bound(c)
    diff = np.abs(_ref(c, W=W - 1) - ref)
    assert (diff > bound).any(axis=(1, 2)).all(), "every row must see the window start"
    # dropping one selected entry is caught too
    sel = c["sel"].copy()
    r = int(np.flatnonzero((sel >= 0).any(1))[-1])
    sel[r, 0] = -1
    diff1 = np.abs(_ref(c, sel=sel)[r] - ref[r])
    assert (diff1 > bound[r]).mean() > 0.1
