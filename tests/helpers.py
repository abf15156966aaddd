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


def quant_codes_match(codes_gpu, codes_orc, pre_values, scales, fmt="fp8", rtol=1e-5):
    """Count code mismatches not explained by a value within rtol of a rounding
    boundary.  pre_values: the oracle's pre-quantisation values; scales: the
    per-element scale (FP8) or 2^X (MXFP4) the oracle used."""
    cg = np.asarray(codes_gpu).reshape(-1)
    co = np.asarray(codes_orc).reshape(-1)
    q = (np.asarray(pre_values, np.float64).reshape(-1) / np.asarray(scales, np.float64).reshape(-1))
    mism = np.flatnonzero(cg != co)
    if mism.size == 0:
        return 0
    dec = (lambda c: np.array([oracle.e4m3_value(int(x)) for x in c])) if fmt == "fp8" else \
          (lambda c: np.array([oracle.e2m1_value(int(x)) for x in c]))
    vg, vo = dec(cg[mism]), dec(co[mism])
    mid = 0.5 * (vg + vo)
    zero_pair = (vg == 0) & (vo == 0)          # +0 / -0
    near = np.abs(q[mism] - mid) <= rtol * np.maximum(np.abs(q[mism]), 1e-30)
    return int((~(near | zero_pair)).sum())
