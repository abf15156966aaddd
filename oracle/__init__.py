"""CPU oracle for the CSA / HCA attention path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does; the two
share no code.  The arithmetic lives in ``csa_oracle.cpp`` (plain loops in
float64); this module only builds it with g++, loads it with ctypes and
marshals numpy arrays.

Format codes: F32=0, BF16=1 (uint16 bits), FP8_S64=2 (uint8 E4M3 codes plus an
fp32 scale per 64 channels), MXFP4=3 (packed E2M1 plus an E8M0 byte per 32
channels), F64=4.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

F32, BF16, FP8_S64, MXFP4, F64 = 0, 1, 2, 3, 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


_NATIVE = os.path.join(_HERE, "liboracle_native.so")


def build(force: bool = False) -> str:
    """Compile the oracle (g++, -O2, OpenMP available but off unless asked)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-fopenmp",
                               _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def build_native() -> str:
    """Compile the same source for timing the CPU baseline on this host:
    -O3 -march=native with OpenMP.  Always rebuilt, since the host's CPU decides
    what -march=native means.  The arithmetic is the same source; only the
    compiler's code generation differs."""
    tmp = _NATIVE + f".tmp{os.getpid()}"
    subprocess.check_call(["g++", "-O3", "-march=native", "-std=c++17", "-shared", "-fPIC",
                           "-fopenmp", _SRC, "-o", tmp])
    os.replace(tmp, _NATIVE)
    return _NATIVE


def use_native() -> None:
    """Load the -O3 -march=native build in place of the parity build (for the
    timed CPU baseline; the parity tests use the default build)."""
    global _lib, _LIB
    build_native()
    _LIB, _lib = _NATIVE, None
    lib()


def lib():
    global _lib
    if _lib is None:
        if _LIB != _NATIVE:
            build()
        L = C.CDLL(_LIB)
        P, I64, I32, D = C.c_void_p, C.c_int64, C.c_int, C.c_double
        L.orc_e4m3_value.restype = D
        L.orc_e4m3_value.argtypes = [C.c_uint8]
        L.orc_e2m1_value.restype = D
        L.orc_e2m1_value.argtypes = [C.c_uint8]
        L.orc_e8m0_value.restype = D
        L.orc_e8m0_value.argtypes = [C.c_uint8]
        L.orc_bf16_value.restype = D
        L.orc_bf16_value.argtypes = [C.c_uint16]
        L.orc_dequantize.argtypes = [I32, P, P, I64, I32, P]
        L.orc_quantize_fp8_s64.argtypes = [P, I64, I32, P, P]
        L.orc_quantize_mxfp4.argtypes = [P, I64, I32, P, P]
        L.orc_compress.argtypes = [I32, P, I32, P, P, I64, I32, I32, P]
        L.orc_f32_to_bf16.argtypes = [P, I64, P]
        L.orc_n_elig.restype = I64
        L.orc_n_elig.argtypes = [I64, I32, I32]
        L.orc_indexer.argtypes = [I32, P, P, P, I32, P, P, I64, P, I64, I32, I32, I32, I32, P, I64, I32]
        L.orc_topk.argtypes = [P, I64, P, I64, I32, I32, I32, P]
        L.orc_attention.argtypes = [I32, P, I32, P, P, I64, P, I32, I32, P, I64, I64, P, P, I64,
                                    I32, I32, I32, I32, D, P, I32]
        L.orc_csa.argtypes = [I32, P, I32, P, P, I32, P, P, P, P, P, I64, I32, P, I64, I64,
                              P, P, I64, I32, I32, I32, I32, I32, I32, I32, D, P, P, I32]
        L.orc_max_threads.restype = I32
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- codecs
def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e8m0_value(code: int) -> float:
    return lib().orc_e8m0_value(code)


def bf16_value(bits: int) -> float:
    return lib().orc_bf16_value(bits)


class Stored:
    """A stored tensor: format code, data array and optional scale array."""

    def __init__(self, fmt, data, scales=None, d=None):
        self.fmt = fmt
        self.data = np.ascontiguousarray(data)
        self.scales = None if scales is None else np.ascontiguousarray(scales)
        self.d = d if d is not None else (self.data.shape[-1] * (2 if fmt == MXFP4 else 1))

    @property
    def rows(self):
        per = self.d // 2 if self.fmt == MXFP4 else self.d
        return self.data.size // per


def dequantize(t: Stored) -> np.ndarray:
    out = np.empty((t.rows, t.d), dtype=np.float64)
    lib().orc_dequantize(t.fmt, _p(t.data), _p(t.scales), t.rows, t.d, _p(out))
    return out


def quantize_fp8_s64(v: np.ndarray) -> Stored:
    v = _c(v, np.float32)
    d = v.shape[-1]
    rows = v.size // d
    codes = np.empty((rows, d), dtype=np.uint8)
    scales = np.empty((rows, d // 64), dtype=np.float32)
    lib().orc_quantize_fp8_s64(_p(v), rows, d, _p(codes), _p(scales))
    return Stored(FP8_S64, codes, scales, d)


def quantize_mxfp4(v: np.ndarray) -> Stored:
    v = _c(v, np.float32)
    d = v.shape[-1]
    rows = v.size // d
    packed = np.zeros((rows, d // 2), dtype=np.uint8)
    sc = np.empty((rows, d // 32), dtype=np.uint8)
    lib().orc_quantize_mxfp4(_p(v), rows, d, _p(packed), _p(sc))
    return Stored(MXFP4, packed, sc, d)


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().orc_f32_to_bf16(_p(v), v.size, _p(out))
    return out


def n_elig(t: int, m: int, W: int) -> int:
    return lib().orc_n_elig(t, m, W)


# ------------------------------------------------------------- method
def compress(x: Stored, z: Stored, bias: np.ndarray, m: int) -> np.ndarray:
    """Pooled entries, fp32 [n_tokens/m][d]."""
    d = x.d
    n = x.rows
    assert n % m == 0 and z.rows == n and z.d == d
    bias = _c(bias, np.float32)
    assert bias.shape == (m, d)
    out = np.empty((n // m, d), dtype=np.float32)
    lib().orc_compress(x.fmt, _p(x.data), z.fmt, _p(z.data), _p(bias), n, m, d, _p(out))
    return out


def indexer(qI: Stored, w: np.ndarray, kI: Stored, q_pos, HI: int, m: int, W: int,
            n_threads: int = 1) -> np.ndarray:
    """Scores [n_q][n_blocks] (fp32); entries beyond n_elig(t) are -inf."""
    q_pos = _c(q_pos, np.int64)
    n_q = q_pos.size
    dI = qI.d
    w = _c(w, np.float32)
    nb = kI.rows
    ld = max(nb, 1)
    out = np.full((n_q, ld), -np.inf, dtype=np.float32)
    ne = np.array([min(n_elig(int(t), m, W), nb) for t in q_pos])
    assert (ne <= nb).all()
    lib().orc_indexer(qI.fmt, _p(qI.data), _p(qI.scales), _p(w), kI.fmt, _p(kI.data),
                      _p(kI.scales), nb, _p(q_pos), n_q, HI, dI, m, W, _p(out), ld, n_threads)
    return out[:, :nb]


def topk(scores: np.ndarray, q_pos, k: int, m: int, W: int) -> np.ndarray:
    scores = _c(scores, np.float32)
    q_pos = _c(q_pos, np.int64)
    rows, ld = scores.shape
    idx = np.empty((rows, k), dtype=np.int32)
    lib().orc_topk(_p(scores), ld, _p(q_pos), rows, k, m, W, _p(idx))
    return idx


def attention(q: Stored, kv: Stored, sel, raw: Stored, raw_pos0: int, sinks, q_pos,
              H: int, m: int, W: int, scale: float, n_threads: int = 1) -> np.ndarray:
    """float64 [n_q][H][d].  sel=None means dense (HCA) over n_elig(t) entries."""
    q_pos = _c(q_pos, np.int64)
    n_q = q_pos.size
    d = q.d
    k = 0 if sel is None else sel.shape[-1]
    sel = _c(sel, np.int32)
    sinks = _c(sinks, np.float32)
    out = np.empty((n_q, H, d), dtype=np.float64)
    lib().orc_attention(q.fmt, _p(q.data), kv.fmt, _p(kv.data), _p(kv.scales), kv.rows, _p(sel), k,
                        raw.fmt, _p(raw.data), raw_pos0, raw.rows, _p(sinks), _p(q_pos), n_q,
                        H, d, m, W, scale, _p(out), n_threads)
    return out


def csa(q: Stored, kv: Stored, qI: Stored, w, kI: Stored, raw: Stored, raw_pos0: int, sinks,
        q_pos, H: int, HI: int, m: int, W: int, k: int, scale: float, n_threads: int = 1):
    """Whole CSA read path for one sequence: (selected ids [n_q][k], out [n_q][H][d])."""
    assert qI.fmt == kI.fmt
    q_pos = _c(q_pos, np.int64)
    n_q = q_pos.size
    d, dI = q.d, qI.d
    w = _c(w, np.float32)
    sinks = _c(sinks, np.float32)
    sel = np.empty((n_q, k), dtype=np.int32)
    out = np.empty((n_q, H, d), dtype=np.float64)
    lib().orc_csa(q.fmt, _p(q.data), kv.fmt, _p(kv.data), _p(kv.scales), qI.fmt, _p(qI.data),
                  _p(qI.scales), _p(w), _p(kI.data), _p(kI.scales), kI.rows, raw.fmt,
                  _p(raw.data), raw_pos0, raw.rows, _p(sinks), _p(q_pos), n_q, H, d, HI, dI, m,
                  W, k, scale, _p(sel), _p(out), n_threads)
    return sel, out


def max_threads() -> int:
    return lib().orc_max_threads()
