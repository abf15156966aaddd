"""Shared test helpers: moving synthetic inputs to the device, building both
sides' stored tensors from the same values, and the matching rules.

Matching rules (written here once, used by every parity test):
  * integer / byte results (top-k ids, quantised codes) are bit-exact, except
    top-k ids whose oracle score lies within 1e-3 relative of the k-th score
    (near-ties), and quantised codes whose oracle pre-quantisation value lies
    within 1e-5 relative of a rounding boundary;
  * fp32 results agree within 1e-5 relative (with an absolute floor of 1e-5
    times the magnitude of the row, for elements that cancel to near zero);
  * bf16 / FP8 results agree within 2e-2 absolute.
"""
from __future__ import annotations

import numpy as np
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth

FMT = {"f32": K.F32, "bf16": K.BF16, "fp8": K.FP8_S64, "mxfp4": K.MXFP4}
ORC_FMT = {"f32": oracle.F32, "bf16": oracle.BF16, "fp8": oracle.FP8_S64, "mxfp4": oracle.MXFP4}


def up(a: np.ndarray, bf16: bool = False) -> torch.Tensor:
    """Host array -> contiguous CUDA tensor (uint16 arrays as bf16 when asked)."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    if bf16:
        t = t.view(torch.bfloat16)
    return t.cuda()


def down(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def act_dev(a: np.ndarray, act: str) -> torch.Tensor:
    return up(a, bf16=(act == "bf16"))


def act_orc(a: np.ndarray, act: str) -> "oracle.Stored":
    a = np.ascontiguousarray(a)
    return oracle.Stored(ORC_FMT[act], a.reshape(-1, a.shape[-1]))


def gpu_quantize(values_f32: np.ndarray, fmt: str) -> "K.Stored":
    """The library's own quantiser applied on the device to fp32 values."""
    d = values_f32.shape[-1]
    rows = values_f32.size // d
    src = up(np.ascontiguousarray(values_f32, np.float32).reshape(rows, d))
    st = K.empty_stored(FMT[fmt], rows, d)
    K.csa_quantize(src, st)
    return st


def orc_quantize(values_f32: np.ndarray, fmt: str) -> "oracle.Stored":
    v = np.ascontiguousarray(values_f32, np.float32)
    v = v.reshape(-1, v.shape[-1])
    if fmt == "fp8":
        return oracle.quantize_fp8_s64(v)
    if fmt == "mxfp4":
        return oracle.quantize_mxfp4(v)
    if fmt == "bf16":
        return oracle.Stored(oracle.BF16, oracle.f32_to_bf16(v))
    return oracle.Stored(oracle.F32, v)


def both_stored(values_f32: np.ndarray, fmt: str):
    """(device Stored from the library quantiser, oracle Stored from its own)."""
    if fmt == "f32":
        v = np.ascontiguousarray(values_f32, np.float32)
        return K.Stored(K.F32, up(v.reshape(-1, v.shape[-1]))), orc_quantize(v, "f32")
    return gpu_quantize(values_f32, fmt), orc_quantize(values_f32, fmt)


def assert_close_f32(got, ref, rtol=1e-5, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    row_mag = np.max(np.abs(ref), axis=-1, keepdims=True) if ref.ndim else np.abs(ref)
    tol = rtol * np.maximum(np.abs(ref), row_mag)
    bad = np.abs(got - ref) > tol
    if bad.any():
        i = np.unravel_index(np.argmax(np.abs(got - ref) - tol), ref.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside rtol {rtol}; "
                             f"worst at {i}: got {got[i]!r} ref {ref[i]!r}")


def assert_close_abs(got, ref, atol=2e-2, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    if not (err <= atol).all():
        i = np.unravel_index(np.argmax(err), ref.shape)
        raise AssertionError(f"{what}: max abs error {err.max():.3g} > {atol} at {i}: "
                             f"got {got[i]!r} ref {ref[i]!r}")


def check_selection(sel_gpu, scores_orc, n_elig, k, rtol=1e-3, what=""):
    """Validate one row's selection: exactly min(k, n) distinct eligible ids,
    ascending, -1 padded, agreeing with the oracle's set except for ids whose
    oracle score lies within rtol * |s_k| of the k-th score s_k."""
    sel_gpu = np.asarray(sel_gpu)
    n = int(n_elig)
    take = min(k, n)
    got = sel_gpu[:take]
    assert np.all(sel_gpu[take:] == -1), f"{what}: padding"
    assert np.all(np.diff(got) > 0), f"{what}: not strictly ascending"
    assert take == 0 or (got[0] >= 0 and got[-1] < n), f"{what}: id out of range"
    if take == 0:
        return
    s = np.asarray(scores_orc[:n], np.float64)
    order = np.lexsort((np.arange(n), -s))
    want = np.sort(order[:take])
    if np.array_equal(got, want):
        return
    sk = s[order[take - 1]]
    band = rtol * abs(sk)
    diff = np.setxor1d(got, want)
    near = np.abs(s[diff] - sk) <= band
    assert near.all(), (f"{what}: {(~near).sum()} selected ids differ beyond the tie band; "
                        f"e.g. id {diff[~near][0]} score {s[diff[~near][0]]} vs k-th {sk}")
    # every id the GPU chose must score at least as high as the band's floor
    assert (s[got] >= sk - band).all(), f"{what}: a selected id scores below the k-th band"


def rounding_flips_ok(got_vals, ref_vals, pre_values, rtol=1e-5):
    """Count stored values that differ between the two sides for a reason other
    than a rounding boundary.  Both sides round their own fp32 pooled value
    once; the fp32 values may differ within the fp32 rule (rtol of
    max(|value|, the row's largest |value|), see assert_close_f32), so the
    stored values may differ only where the oracle's pre-rounding value lies
    within that distance of the midpoint between the two stored values.
    Arrays are [rows][d] in value units (the stored value, scale applied)."""
    vg = np.asarray(got_vals, np.float64)
    vo = np.asarray(ref_vals, np.float64)
    pre = np.asarray(pre_values, np.float64)
    tol = rtol * np.maximum(np.abs(pre), np.max(np.abs(pre), axis=-1, keepdims=True))
    mism = vg != vo
    if not mism.any():
        return 0
    near = np.abs(pre - 0.5 * (vg + vo)) <= tol
    return int((mism & ~near).sum())


def quant_codes_match(codes_gpu, codes_orc, pre_values, scales, fmt="fp8", rtol=1e-5):
    """Count code mismatches not explained by a value near a rounding boundary
    (rounding_flips_ok on the decoded values).  codes [rows][d] (MXFP4:
    unpacked nibbles); pre_values: the oracle's pre-quantisation values;
    scales: the per-element scale (FP8) or 2^X (MXFP4) the oracle used."""
    cg = np.asarray(codes_gpu)
    co = np.asarray(codes_orc)
    sc = np.asarray(scales, np.float64)
    table = np.array([oracle.e4m3_value(i) for i in range(256)]) if fmt == "fp8" else \
        np.array([oracle.e2m1_value(i) for i in range(16)])
    return rounding_flips_ok(table[cg] * sc, table[co] * sc, pre_values, rtol)


def bf16_values_match(got_bits, ref_bits, pre_values, rtol=1e-5):
    """Count bf16 values that differ for a reason other than a rounding boundary."""
    g = synth.bf16_bits_to_f32_np(np.asarray(got_bits, np.uint16))
    r = synth.bf16_bits_to_f32_np(np.asarray(ref_bits, np.uint16))
    return rounding_flips_ok(g, r, pre_values, rtol)


# ------------------------------------------------------------------ attention
# A second, tighter tolerance for the tensor-core attention paths, derived from
# the arithmetic those kernels perform (on top of the 2e-2 absolute rule):
#   * each dequantised FP8 entry value (E4M3 x fp32 scale) is rounded once to
#     bf16 before it is used as key and value (relative error <= u = 2^-9);
#     bf16-stored entries, window tokens and q are used exactly;
#   * each softmax probability P is rounded once to bf16 (relative <= u);
#   * dot products and the P.V sums accumulate in fp32, and the output is
#     rounded once to bf16.
# First-order propagation gives, for output o[h][c] = sum_e p_e v_ec / L,
#   do = sum_{e,i} a_{e,i} eps_{e,i} + sum_e b_e eta_e
#   a_{e,i} = (p_e/L) [ (v_ec - o_hc) scale q_hi k_ei + [i = c] v_ec ]   (entry roundings)
#   b_e     = (p_e/L) v_ec                                                (P roundings)
# with |eps|, |eta| <= u.  Under the probabilistic model of rounding errors
# (independent, mean zero: N. J. Higham and T. Mary, "A new approach to
# probabilistic rounding error analysis", SIAM J. Sci. Comput. 41 (2019)),
# Hoeffding's inequality bounds |do| by lam * u * sqrt(sum a^2 + sum b^2)
# except with probability 2 exp(-lam^2 / 2) (lam = 8: 2.5e-14 per element).
# (sum a^2 is bounded with (x + y)^2 <= 2x^2 + 2y^2.)  Deterministic terms are
# added for the output rounding (u |o|), the fp32 accumulation of the D-long
# logits (D 2^-24 scale sum_i |q_i k_i|) and of the P.V sums (n 2^-24 sum p|v|).
U_BF16 = 2.0 ** -9
U_F32 = 2.0 ** -24


def attention_items(t, n_ent, sel_row, m, W, raw_pos0, n_raw):
    """(entry ids, window positions) attended by the query at position t:
    the selected ids (or every visible entry when sel_row is None) and the
    raw positions t-W < pos <= t held by the raw buffer."""
    ne = min(max(0, (t - W) // m) if t - W > 0 else 0, n_ent)
    if sel_row is None:
        ids = np.arange(ne)
    else:
        s = np.asarray(sel_row)
        ids = s[(s >= 0) & (s < n_ent)]
    lo = max(t - W + 1, 0, raw_pos0)
    hi = min(t, raw_pos0 + n_raw - 1)
    pos = np.arange(lo, hi + 1) if hi >= lo else np.zeros(0, np.int64)
    return ids, pos


def attention_bound(q, ent, ent_rounded, sel, raw, raw_pos0, sinks, q_pos, m, W, scale,
                    lam=8.0):
    """Per-element tolerance [n_q][H][d] for a bf16 tensor-core attention
    output (see the derivation above).  q [n_q][H][d], ent [n_ent][d] and
    raw [n_raw][d] are the float values of the stored inputs (dequantised);
    ent_rounded: whether the kernel rounds entry values to bf16 (FP8 entries)."""
    q = np.asarray(q, np.float64)
    ent = np.asarray(ent, np.float64)
    raw = np.asarray(raw, np.float64)
    n_q, H, d = q.shape
    out = np.empty((n_q, H, d))
    for r in range(n_q):
        t = int(q_pos[r])
        ids, pos = attention_items(t, ent.shape[0], None if sel is None else sel[r], m, W,
                                   raw_pos0, raw.shape[0])
        K = np.concatenate([ent[ids], raw[pos - raw_pos0]], 0)
        rnd = np.concatenate([np.full(len(ids), bool(ent_rounded)), np.zeros(len(pos), bool)])
        qr = q[r]
        lg = scale * qr @ K.T                                   # [H][E]
        M = lg.max(1) if K.shape[0] else np.full(H, -np.inf)
        if sinks is not None:
            M = np.maximum(M, np.asarray(sinks, np.float64))
        p = np.exp(lg - M[:, None])
        L = p.sum(1) + (np.exp(np.asarray(sinks, np.float64) - M) if sinks is not None else 0.0)
        P = p / L[:, None]
        o = P @ K                                               # [H][d]
        K2, Ka = K * K, np.abs(K)
        # entry roundings: 2 scale^2 sum_e c_he (v_ec - o_hc)^2 + 2 sum_e w_he v_ec^2
        w = (P * P) * rnd[None, :]
        c = w * ((qr * qr) @ K2.T)
        a = 2 * scale * scale * (c @ K2 - 2 * o * (c @ K) + o * o * c.sum(1)[:, None]) + 2 * (w @ K2)
        b = (P * P) @ K2                                        # P roundings
        A = scale * np.abs(qr) @ Ka.T                           # scale sum_i |q_i k_i|
        det = (d * U_F32 * ((P * A) @ Ka + np.abs(o) * (P * A).sum(1)[:, None])
               + K.shape[0] * U_F32 * (P @ Ka))
        out[r] = lam * U_BF16 * np.sqrt(np.maximum(a, 0.0) + b) + U_BF16 * np.abs(o) + det + 1e-7
    return out


def assert_within_bound(got, ref, bound, what=""):
    """Element-wise |got - ref| <= bound (the arithmetic-derived tolerance)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err / bound), ref.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside the derived bound; "
                             f"worst at {i}: err {err[i]:.3g} bound {bound[i]:.3g} "
                             f"(got {got[i]!r} ref {ref[i]!r}); max err/bound {np.max(err / bound):.3g}")


def assert_attention_close(got, ref, bound, what=""):
    """Both matching rules of the bf16 / FP8 attention outputs: the 2e-2
    absolute rule and the arithmetic-derived element bound."""
    assert_close_abs(got, ref, 2e-2, what)
    assert_within_bound(got, ref, bound, what)


def stored_values(st) -> np.ndarray:
    """Float values (float64) of an oracle Stored tensor, by the oracle's own decoder."""
    return oracle.dequantize(st)


def attention_bound_stored(q_st, kv_st, sel, raw_st, raw_pos0, sinks, q_pos, H, m, W, scale):
    """attention_bound on oracle-stored inputs: q [n_q * H][d], entries, raw."""
    q_pos = np.asarray(q_pos, np.int64).reshape(-1)
    qv = stored_values(q_st).reshape(q_pos.size, H, -1)
    return attention_bound(qv, stored_values(kv_st), kv_st.fmt == oracle.FP8_S64, sel,
                           stored_values(raw_st), raw_pos0, sinks, q_pos, m, W, scale)


def sink_dominant(q_st, kv_st, sel, raw_st, raw_pos0, q_pos, H, m, W, scale, shift=2.0):
    """Per-head sink logits `shift` above the largest logit any of the given
    queries attends: the sink then dominates every softmax denominator, so a
    kernel that mishandles it fails both matching rules."""
    q_pos = np.asarray(q_pos, np.int64).reshape(-1)
    qv = stored_values(q_st).reshape(q_pos.size, H, -1)
    ent, raw = stored_values(kv_st), stored_values(raw_st)
    mx = np.full(H, -1e30)
    for r, t in enumerate(q_pos):
        ids, pos = attention_items(int(t), ent.shape[0], None if sel is None else sel[r], m, W,
                                   raw_pos0, raw.shape[0])
        K = np.concatenate([ent[ids], raw[pos - raw_pos0]], 0)
        if K.shape[0]:
            mx = np.maximum(mx, (scale * qv[r] @ K.T).max(1))
    return (mx + shift).astype(np.float32)
