"""B200 (sm_100a) library for DeepSeek-V4's hybrid attention (CSA + HCA).

This module is the thin Python binding of ``libcsa13.so`` (C ABI declared in
``include/csa.h``).  It only marshals arguments: torch tensors supply device
memory and streams, every computation runs in the library's CUDA kernels.
Importing works without a GPU (the library loads, nothing launches); calling
anything without the built library raises.

Names follow the C ABI: ``csa_compress``, ``csa_quantize``, ``indexer_score``,
``topk_select``, ``sparse_mqa_attn``, ``hca_attn``, ``window_attn``, ``csa_decode``,
``csa_prefill``, ``csa_workspace_size``, ``csa_device_status``, and
``csa_decode_noalloc`` (csa_decode on the library's fixed device scratch, for
callers that cannot allocate).
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass

F32, BF16, FP8_S64, MXFP4 = 0, 1, 2, 3
OP_SPARSE_ATTN, OP_HCA_ATTN, OP_DECODE, OP_PREFILL, OP_WINDOW_ATTN = 0, 1, 2, 3, 4
OP_SHARD_SELECT, OP_SHARD_ATTEND, OP_HCA_SHARD = 5, 6, 7
FLAG_BATCH_INVARIANT = 0x1
FLAG_QI_BF16 = 0x2
FLAG_INDEXER_FP8 = 0x4
DEV_BAD_INDEX, DEV_RANGE, DEV_TIMEOUT = 0x1, 0x2, 0x4
NOALLOC_SCRATCH_BYTES = 32 << 20   # CSA_NOALLOC_SCRATCH_BYTES
ERR_WORKSPACE = -4

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa13.so")
_lib = None


class CsaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({strerror(status)})")


class Params(C.Structure):
    """Mirror of ``csa_params``."""
    _fields_ = [("m", C.c_int32), ("window", C.c_int32), ("top_k", C.c_int32),
                ("n_heads", C.c_int32), ("head_dim", C.c_int32), ("idx_heads", C.c_int32),
                ("idx_dim", C.c_int32), ("scale", C.c_float), ("act_fmt", C.c_int32),
                ("kv_fmt", C.c_int32), ("idx_fmt", C.c_int32), ("flags", C.c_uint32)]


def params(m, window, top_k, n_heads, head_dim, idx_heads, idx_dim, scale,
           act_fmt=BF16, kv_fmt=FP8_S64, idx_fmt=MXFP4, flags=0) -> Params:
    return Params(m, window, top_k, n_heads, head_dim, idx_heads, idx_dim, float(scale),
                  act_fmt, kv_fmt, idx_fmt, flags)


EXPORTS = ["csa_compress", "csa_quantize", "indexer_score", "topk_select", "sparse_mqa_attn",
           "hca_attn", "window_attn", "csa_decode", "csa_prefill", "csa_workspace_size",
           "csa_device_status", "csa_strerror", "csa_version", "csa_decode_noalloc",
           "csa_shard_select", "csa_shard_attend", "hca_shard_attend", "attn_merge"]


def lib():
    """Load libcsa13.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m compressed_sparse_attention_13_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, I32, I64, PP = C.c_void_p, C.c_int32, C.c_int64, C.POINTER(Params)
        L.csa_compress.argtypes = [PP, I32, P, P, P, I64, I32, P, P, P]
        L.csa_quantize.argtypes = [I32, P, I64, I32, P, P, P]
        L.indexer_score.argtypes = [PP, I32, I32, P, P, P, P, P, I64, P, P, I64, P]
        L.topk_select.argtypes = [PP, I32, I32, P, I64, I64, P, P, P]
        L.sparse_mqa_attn.argtypes = [PP, I32, I32, P, P, P, I64, P, P, I64, P, P, P, P, P,
                                      C.c_size_t, P]
        L.hca_attn.argtypes = [PP, I32, I32, P, P, P, I64, P, I64, P, P, P, P, P, C.c_size_t, P]
        L.window_attn.argtypes = [PP, I32, I32, P, P, I64, P, P, P, P, P, C.c_size_t, P]
        L.csa_decode.argtypes = [PP, I32, P, P, P, P, P, P, P, P, I64, P, I64, P, P, P, P, P, P,
                                 C.c_size_t, P]
        L.csa_prefill.argtypes = [PP, I32, I64, I64, P, I64, I64, P, P, P, P, P, P, P, P, P, P,
                                  I64, P, P, P, P, C.c_size_t, P]
        L.csa_decode_noalloc.argtypes = [PP, I32, P, P, P, P, P, P, P, P, I64, P, I64, P, P, P,
                                         P, P, P]
        L.csa_shard_select.argtypes = [PP, I32, P, P, P, P, P, I64, I64, P, P, P, P, C.c_size_t, P]
        L.csa_shard_attend.argtypes = [PP, I32, P, I32, P, P, P, P, I64, I64, P, I64, P, P, P, P, P, P,
                                       C.c_size_t, P]
        L.hca_shard_attend.argtypes = [PP, I32, P, P, P, I64, I64, P, I64, P, P, P, P, P, C.c_size_t, P]
        L.attn_merge.argtypes = [PP, I32, I32, P, P, P, P, P]
        L.csa_workspace_size.restype = C.c_size_t
        L.csa_workspace_size.argtypes = [PP, I32, I32, I64, I64]
        L.csa_device_status.argtypes = [P, C.POINTER(C.c_uint32), I32]
        L.csa_strerror.restype = C.c_char_p
        L.csa_strerror.argtypes = [C.c_int]
        L.csa_version.restype = C.c_char_p
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().csa_strerror(status).decode()


def version() -> str:
    return lib().csa_version().decode()


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _s(stream):
    import torch
    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _ok(fn, st):
    if st != 0:
        raise CsaError(fn, st)


@dataclass
class Stored:
    """A stored tensor: data plus per-group scales (FP8_S64 / MXFP4)."""
    fmt: int
    data: "object"
    scales: "object" = None


def empty_stored(fmt: int, rows: int, d: int, device="cuda") -> Stored:
    """Allocate (with torch) a [rows][d] tensor in a stored format."""
    import torch
    if fmt == F32:
        return Stored(fmt, torch.empty(rows, d, dtype=torch.float32, device=device))
    if fmt == BF16:
        return Stored(fmt, torch.empty(rows, d, dtype=torch.bfloat16, device=device))
    if fmt == FP8_S64:
        return Stored(fmt, torch.empty(rows, d, dtype=torch.uint8, device=device),
                      torch.empty(rows, d // 64, dtype=torch.float32, device=device))
    if fmt == MXFP4:
        return Stored(fmt, torch.empty(rows, d // 2, dtype=torch.uint8, device=device),
                      torch.empty(rows, d // 32, dtype=torch.uint8, device=device))
    raise ValueError(fmt)


# --------------------------------------------------------------- entry points
def csa_compress(p: Params, d: int, x, z, bias, n_tokens: int, out: Stored, stream=None):
    _ok("csa_compress", lib().csa_compress(C.byref(p), d, _p(x), _p(z), _p(bias), n_tokens,
                                           out.fmt, _p(out.data), _p(out.scales), _s(stream)))


def csa_quantize(src, out: Stored, stream=None):
    d = src.shape[-1]
    rows = src.numel() // d
    _ok("csa_quantize", lib().csa_quantize(out.fmt, _p(src), rows, d, _p(out.data),
                                           _p(out.scales), _s(stream)))


def indexer_score(p: Params, batch: int, n_q: int, qI: Stored, w, kI: Stored, max_blocks: int,
                  q_pos, scores, ld_scores: int, stream=None):
    _ok("indexer_score", lib().indexer_score(
        C.byref(p), batch, n_q, _p(qI.data), _p(qI.scales), _p(w), _p(kI.data), _p(kI.scales),
        max_blocks, _p(q_pos), _p(scores), ld_scores, _s(stream)))


def topk_select(p: Params, batch: int, n_q: int, scores, ld_scores: int, max_blocks: int, q_pos,
                idx, stream=None):
    _ok("topk_select", lib().topk_select(C.byref(p), batch, n_q, _p(scores), ld_scores,
                                         max_blocks, _p(q_pos), _p(idx), _s(stream)))


def csa_workspace_size(p: Params, op: int, batch: int, n_q: int, n_ctx: int) -> int:
    return lib().csa_workspace_size(C.byref(p), op, batch, n_q, n_ctx)


def _ws(ws):
    return (None, 0) if ws is None else (_p(ws), ws.numel() * ws.element_size())


def sparse_mqa_attn(p: Params, batch: int, n_q: int, q, kv: Stored, max_entries: int, idx, raw,
                    n_raw: int, raw_pos0, q_pos, sinks, out, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _ok("sparse_mqa_attn", lib().sparse_mqa_attn(
        C.byref(p), batch, n_q, _p(q), _p(kv.data), _p(kv.scales), max_entries, _p(idx), _p(raw),
        n_raw, _p(raw_pos0), _p(q_pos), _p(sinks), _p(out), wp, wb, _s(stream)))


def hca_attn(p: Params, batch: int, n_q: int, q, kv: Stored, max_entries: int, raw, n_raw: int,
             raw_pos0, q_pos, sinks, out, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _ok("hca_attn", lib().hca_attn(
        C.byref(p), batch, n_q, _p(q), _p(kv.data), _p(kv.scales), max_entries, _p(raw), n_raw,
        _p(raw_pos0), _p(q_pos), _p(sinks), _p(out), wp, wb, _s(stream)))


def window_attn(p: Params, batch: int, n_q: int, q, raw, n_raw: int, raw_pos0, q_pos, sinks, out,
                workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _ok("window_attn", lib().window_attn(
        C.byref(p), batch, n_q, _p(q), _p(raw), n_raw, _p(raw_pos0), _p(q_pos), _p(sinks), _p(out),
        wp, wb, _s(stream)))


def csa_decode(p: Params, batch: int, q, qI: Stored, w, kv: Stored, kI: Stored, max_blocks: int,
               raw, n_raw: int, raw_pos0, q_pos, sinks, out, idx_out, workspace, stream=None):
    wp, wb = _ws(workspace)
    _ok("csa_decode", lib().csa_decode(
        C.byref(p), batch, _p(q), _p(qI.data), _p(qI.scales), _p(w), _p(kv.data), _p(kv.scales),
        _p(kI.data), _p(kI.scales), max_blocks, _p(raw), n_raw, _p(raw_pos0), _p(q_pos),
        _p(sinks), _p(out), _p(idx_out), wp, wb, _s(stream)))


def csa_decode_noalloc(p: Params, batch: int, q, qI: Stored, w, kv: Stored, kI: Stored,
                       max_blocks: int, raw, n_raw: int, raw_pos0, q_pos, sinks, out, idx_out,
                       stream=None):
    """csa_decode without a workspace argument: the library's fixed device scratch
    is used instead.  Calls on one device must not overlap; requests larger than
    NOALLOC_SCRATCH_BYTES raise CsaError with status ERR_WORKSPACE."""
    _ok("csa_decode_noalloc", lib().csa_decode_noalloc(
        C.byref(p), batch, _p(q), _p(qI.data), _p(qI.scales), _p(w), _p(kv.data), _p(kv.scales),
        _p(kI.data), _p(kI.scales), max_blocks, _p(raw), n_raw, _p(raw_pos0), _p(q_pos),
        _p(sinks), _p(out), _p(idx_out), _s(stream)))


def csa_prefill(p: Params, batch: int, T: int, t0: int, raw, n_raw: int, raw_pos0: int, z, bias,
                q, qI: Stored, w, kv: Stored, kI: Stored, max_blocks: int, sinks, out, idx_out,
                workspace, stream=None):
    wp, wb = _ws(workspace)
    _ok("csa_prefill", lib().csa_prefill(
        C.byref(p), batch, T, t0, _p(raw), n_raw, raw_pos0, _p(z), _p(bias), _p(q), _p(qI.data),
        _p(qI.scales), _p(w), _p(kv.data), _p(kv.scales), _p(kI.data), _p(kI.scales),
        max_blocks, _p(sinks), _p(out), _p(idx_out), wp, wb, _s(stream)))


def csa_shard_select(p: Params, batch: int, qI: Stored, w, kI: Stored, n_entries: int, entry0: int, q_pos,
                     cand_scores, cand_ids, workspace, stream=None):
    wp, wb = _ws(workspace)
    _ok("csa_shard_select", lib().csa_shard_select(
        C.byref(p), batch, _p(qI.data), _p(qI.scales), _p(w), _p(kI.data), _p(kI.scales), n_entries, entry0,
        _p(q_pos), _p(cand_scores), _p(cand_ids), wp, wb, _s(stream)))


def csa_shard_attend(p: Params, batch: int, q, n_parts: int, cand_scores, cand_ids, kv: Stored,
                     n_entries: int, entry0: int, raw, n_raw: int, raw_pos0, q_pos, part_o, part_ml,
                     idx_out, workspace, stream=None):
    wp, wb = _ws(workspace)
    _ok("csa_shard_attend", lib().csa_shard_attend(
        C.byref(p), batch, _p(q), n_parts, _p(cand_scores), _p(cand_ids), _p(kv.data), _p(kv.scales),
        n_entries, entry0, _p(raw), n_raw, _p(raw_pos0), _p(q_pos), _p(part_o), _p(part_ml), _p(idx_out),
        wp, wb, _s(stream)))


def hca_shard_attend(p: Params, batch: int, q, kv: Stored, n_entries: int, entry0: int, raw, n_raw: int,
                     raw_pos0, q_pos, part_o, part_ml, workspace, stream=None):
    wp, wb = _ws(workspace)
    _ok("hca_shard_attend", lib().hca_shard_attend(
        C.byref(p), batch, _p(q), _p(kv.data), _p(kv.scales), n_entries, entry0, _p(raw), n_raw,
        _p(raw_pos0), _p(q_pos), _p(part_o), _p(part_ml), wp, wb, _s(stream)))


def attn_merge(p: Params, batch: int, n_parts: int, part_o, part_ml, sinks, out, stream=None):
    _ok("attn_merge", lib().attn_merge(C.byref(p), batch, n_parts, _p(part_o), _p(part_ml), _p(sinks),
                                       _p(out), _s(stream)))


def csa_device_status(reset: bool = True, stream=None) -> int:
    flags = C.c_uint32(0)
    _ok("csa_device_status", lib().csa_device_status(_s(stream), C.byref(flags), int(reset)))
    return flags.value
