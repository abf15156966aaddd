"""The C-ABI library: it loads without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything."""
import ctypes as C
import os
import re

import pytest

import compressed_sparse_attention_13_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        with open(os.path.join(ROOT, "include", fn)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", src, re.M):
            if m.group(1) not in ("if", "sizeof", "defined"):
                names.add(m.group(1))
    return names


def test_header_declares_the_entry_points():
    want = {"csa_compress", "csa_quantize", "indexer_score", "topk_select", "sparse_mqa_attn",
            "hca_attn", "window_attn", "csa_decode", "csa_prefill", "csa_workspace_size",
            "csa_device_status", "csa_strerror", "csa_version"}
    assert want <= _declared()


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(K.LIB_PATH)
    missing = [n for n in sorted(_declared()) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(K.EXPORTS) <= _declared()


def test_version_and_errors():
    assert "sm_100a" in K.version()
    for st in (0, -1, -2, -3, -4, -5):
        assert K.strerror(st)
    assert K.strerror(-99) == "unknown status"


def test_workspace_size_contract():
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    assert K.csa_workspace_size(p, K.OP_DECODE, 32, 1, 32768) > 32 * 32768 * 4
    assert K.csa_workspace_size(p, 99, 1, 1, 1) == 0
    bad = K.params(4, 128, 512, 0, 512, 64, 128, 0.044)
    assert K.csa_workspace_size(bad, K.OP_DECODE, 1, 1, 1) == 0


def _call(fn, *args):
    return getattr(K.lib(), fn)(*args)


def test_host_side_argument_errors_need_no_gpu():
    """Bad arguments are rejected before any CUDA call, so these run on CPU."""
    lib = K.lib()
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    P = C.byref(p)
    fake = C.c_void_p(0x1000)         # aligned, never dereferenced on the error paths
    odd = C.c_void_p(0x1001)          # misaligned
    # d not a multiple of 64
    assert lib.csa_compress(P, 63, fake, fake, fake, 4, K.F32, fake, None, None) == -1
    # token count not a multiple of m
    assert lib.csa_compress(P, 64, fake, fake, fake, 6, K.F32, fake, None, None) == -1
    # FP8 output without a scale buffer
    assert lib.csa_compress(P, 64, fake, fake, fake, 8, K.FP8_S64, fake, None, None) == -1
    # misaligned input
    assert lib.csa_compress(P, 64, odd, fake, fake, 8, K.F32, fake, None, None) == -2
    # FP8 scales must be 4-byte aligned (MXFP4 scales are single bytes: any address)
    assert lib.csa_compress(P, 64, fake, fake, fake, 8, K.FP8_S64, fake, C.c_void_p(0x1002), None) == -2
    # unknown quantisation format
    assert lib.csa_quantize(7, fake, 4, 64, fake, fake, None) == -1
    # ld_scores smaller than max_blocks
    assert lib.indexer_score(P, 1, 1, fake, fake, fake, fake, fake, 100, fake, fake, 50, None) == -1
    # MXFP4 indexer without scales
    assert lib.indexer_score(P, 1, 1, fake, None, fake, fake, None, 100, fake, fake, 100, None) == -1
    # null selection for sparse attention
    assert lib.sparse_mqa_attn(P, 1, 1, fake, fake, fake, 10, None, fake, 8, fake, fake, None,
                               fake, fake, 1 << 30, None) == -1
    # decode with a too-small workspace
    assert lib.csa_decode(P, 32, fake, fake, fake, fake, fake, fake, fake, fake, 32768, fake, 128,
                          fake, fake, None, fake, None, fake, 16, None) == -4
    # prefill chunk start not a multiple of m
    assert lib.csa_prefill(P, 1, 64, 3, fake, 64, 0, fake, fake, fake, fake, fake, fake, fake,
                           fake, fake, fake, 100, None, fake, None, fake, 1 << 30, None) == -1
    # bad parameter values
    badp = K.params(0, 128, 512, 64, 512, 64, 128, 0.044)
    assert lib.topk_select(C.byref(badp), 1, 1, fake, 10, 10, fake, fake, None) == -1
    nanp = K.params(4, 128, 512, 64, 512, 64, 128, float("nan"))
    assert lib.hca_attn(C.byref(nanp), 1, 1, fake, fake, fake, 10, fake, 8, fake, fake, None,
                        fake, fake, 1 << 20, None) == -1


def test_unbuilt_library_fails_loudly(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(K, "_lib", None)
    monkeypatch.setattr(K, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        K.lib()


def test_empty_inputs_are_no_ops_without_a_gpu():
    """Zero tokens, rows or sequences: every entry point returns 0 before any
    CUDA call (these run on CPU, where a CUDA call would fail)."""
    lib = K.lib()
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    P = C.byref(p)
    fake = C.c_void_p(0x1000)
    assert lib.csa_compress(P, 64, fake, fake, fake, 0, K.F32, fake, None, None) == 0
    assert lib.csa_quantize(K.FP8_S64, fake, 0, 64, fake, fake, None) == 0
    assert lib.indexer_score(P, 0, 1, fake, fake, fake, fake, fake, 100, fake, fake, 100, None) == 0
    assert lib.indexer_score(P, 1, 0, fake, fake, fake, fake, fake, 100, fake, fake, 100, None) == 0
    assert lib.topk_select(P, 0, 1, fake, 10, 10, fake, fake, None) == 0
    assert lib.topk_select(P, 1, 0, fake, 10, 10, fake, fake, None) == 0
    assert lib.sparse_mqa_attn(P, 0, 1, fake, fake, fake, 10, fake, fake, 8, fake, fake, fake,
                               fake, fake, 1 << 20, None) == 0
    assert lib.hca_attn(P, 1, 0, fake, fake, fake, 10, fake, 8, fake, fake, fake,
                        fake, fake, 1 << 20, None) == 0
    assert lib.csa_decode(P, 0, fake, fake, fake, fake, fake, fake, fake, fake, 32768, fake, 128,
                          fake, fake, fake, fake, fake, fake, 1 << 30, None) == 0
    assert lib.csa_prefill(P, 1, 0, 0, fake, 64, 0, fake, fake, fake, fake, fake, fake, fake,
                           fake, fake, fake, 100, fake, fake, fake, fake, 1 << 30, None) == 0
    # sizes beyond size_t saturate, so no buffer passes the workspace check
    assert lib.csa_workspace_size(P, K.OP_PREFILL, 1 << 30, 1 << 40, 1 << 40) == 2 ** 64 - 1
    assert lib.csa_prefill(P, 1 << 30, 1 << 30, 0, fake, 1 << 31, 0, fake, fake, fake, fake, fake,
                           fake, fake, fake, fake, fake, 1 << 30, fake, fake, fake, fake,
                           1 << 40, None) in (-1, -3, -4)
    # workspace queries for empty batches plan no split (this once divided by zero)
    for op in (K.OP_DECODE, K.OP_PREFILL, K.OP_SPARSE_ATTN, K.OP_HCA_ATTN, K.OP_WINDOW_ATTN):
        assert 0 < lib.csa_workspace_size(P, op, 0, 1, 32768) < (1 << 20)
        assert 0 < lib.csa_workspace_size(P, op, 3, 0, 32768) < (1 << 20)
    assert lib.window_attn(P, 0, 1, fake, fake, 8, fake, fake, None, fake, fake, 1 << 20, None) == 0
    assert lib.window_attn(P, 2, 0, fake, fake, 8, fake, fake, None, fake, fake, 1 << 20, None) == 0


def test_cuda_core_paths_refuse_more_rows_than_the_grid_holds():
    """f32 attention and the CUDA-core indexer put query rows on the grid's y
    axis (at most 65535): larger calls are refused on the host."""
    lib = K.lib()
    p = K.params(4, 64, 16, 8, 64, 4, 32, 0.125, act_fmt=K.F32, kv_fmt=K.F32, idx_fmt=K.F32)
    P = C.byref(p)
    fake = C.c_void_p(0x1000)
    assert lib.sparse_mqa_attn(P, 2, 40000, fake, fake, None, 100, fake, fake, 8, fake, fake, None,
                               fake, fake, 1 << 40, None) == -3
    assert lib.indexer_score(P, 2, 40000, fake, None, fake, fake, None, 100, fake, fake, 100, None) == -3


def test_window_attn_and_flags_host_errors():
    lib = K.lib()
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    P = C.byref(p)
    fake, odd = C.c_void_p(0x1000), C.c_void_p(0x1001)
    # no query, no positions, a raw buffer without data, a misaligned output
    assert lib.window_attn(P, 1, 1, None, fake, 8, fake, fake, None, fake, fake, 1 << 20, None) == -1
    assert lib.window_attn(P, 1, 1, fake, fake, 8, fake, None, None, fake, fake, 1 << 20, None) == -1
    assert lib.window_attn(P, 1, 1, fake, None, 8, fake, fake, None, fake, fake, 1 << 20, None) == -1
    assert lib.window_attn(P, 1, 1, fake, fake, 8, fake, fake, None, odd, fake, 1 << 20, None) == -2
    # a workspace below the plan (32 rows of a 128-token window split in two)
    need = lib.csa_workspace_size(P, K.OP_WINDOW_ATTN, 32, 1, 0)
    assert need > 32 * 64 * 512 * 4
    assert lib.window_attn(P, 32, 1, fake, fake, 128, fake, fake, None, fake, fake, 16, None) == -4
    # unknown flag bits are refused
    bad = K.params(4, 128, 512, 64, 512, 64, 128, 0.044, flags=0x80)
    assert lib.hca_attn(C.byref(bad), 1, 1, fake, fake, fake, 10, fake, 8, fake, fake, None,
                        fake, fake, 1 << 20, None) == -1


def test_batch_invariant_plan_depends_on_the_row_only():
    """With CSA_FLAG_BATCH_INVARIANT the attention workspace grows exactly in
    proportion to the rows (the split count per row is fixed), while the
    default plan splits few rows more finely than many."""
    inv = K.params(4, 128, 512, 64, 512, 64, 128, 0.044, flags=K.FLAG_BATCH_INVARIANT)
    dft = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    ws = lambda p, b: K.csa_workspace_size(p, K.OP_SPARSE_ATTN, b, 1, 0) - 256
    assert ws(inv, 32) == 32 * ws(inv, 1)
    assert ws(dft, 1) > ws(dft, 32) / 32


def test_indexer_write_path_flags_host_errors():
    """CSA_FLAG_QI_BF16 / CSA_FLAG_INDEXER_FP8 belong to the MXFP4 indexer:
    another index format is an argument error; with the bf16 query flag the
    query scales are not needed, without it they are; shapes the tensor-core
    indexer does not take are refused before anything is launched."""
    lib = K.lib()
    fake = C.c_void_p(0x1000)
    for flags in (K.FLAG_QI_BF16, K.FLAG_INDEXER_FP8, K.FLAG_QI_BF16 | K.FLAG_INDEXER_FP8):
        bf = K.params(4, 128, 512, 64, 512, 64, 128, 0.044, idx_fmt=K.BF16, flags=flags)
        assert lib.indexer_score(C.byref(bf), 1, 1, fake, None, fake, fake, None, 256, fake, fake, 256,
                                 None) == -1
        # 32 index heads: no tensor-core MXFP4 indexer (query scales given, so only the shape fails)
        p32 = K.params(4, 128, 512, 64, 512, 32, 128, 0.044, idx_fmt=K.MXFP4, flags=flags)
        assert lib.indexer_score(C.byref(p32), 1, 1, fake, fake, fake, fake, fake, 256, fake, fake, 256,
                                 None) == -3
    # the stored-query path needs the query scales; the bf16 query path does not
    # (it reaches the launch check of a 129-key row, not a multiple of 4)
    mx = K.params(4, 128, 512, 64, 512, 64, 128, 0.044, idx_fmt=K.MXFP4)
    assert lib.indexer_score(C.byref(mx), 1, 1, fake, None, fake, fake, fake, 129, fake, fake, 129,
                             None) == -1
    qb = K.params(4, 128, 512, 64, 512, 64, 128, 0.044, idx_fmt=K.MXFP4, flags=K.FLAG_QI_BF16)
    assert lib.indexer_score(C.byref(qb), 1, 1, fake, None, fake, fake, fake, 129, fake, fake, 129,
                             None) == -3


def test_sharded_decode_host_errors():
    """Argument checks of the sharded entry points, before any launch."""
    lib = K.lib()
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    P = C.byref(p)
    fake = C.c_void_p(0x1000)
    # select: negative entry offset; a workspace below the plan
    assert lib.csa_shard_select(P, 1, fake, fake, fake, fake, fake, 1024, -1, fake, fake, fake, fake,
                                1 << 20, None) == -1
    need = lib.csa_workspace_size(P, K.OP_SHARD_SELECT, 2, 1, 4096)
    assert need >= 2 * 4096 * 4 + 2 * 512 * 4
    assert lib.csa_shard_select(P, 2, fake, fake, fake, fake, fake, 4096, 0, fake, fake, fake, fake,
                                need - 1, None) == -4
    # attend: no parts; too many candidates for the merge; no partial output
    args = lambda n_parts, pml: (P, 1, fake, n_parts, fake, fake, fake, fake, 1024, 0, None, 0, fake, fake,
                                 fake, pml, None, fake, 1 << 30, None)
    assert lib.csa_shard_attend(*args(0, fake)) == -1
    assert lib.csa_shard_attend(*args(33, fake)) == -3      # 33 x 512 > 16384 candidates
    assert lib.csa_shard_attend(*args(4, None)) == -1
    # HCA partial without its (M, L) output; merge over no or too many parts
    assert lib.hca_shard_attend(P, 1, fake, fake, fake, 1024, 0, None, 0, fake, fake, fake, None, fake,
                                1 << 30, None) == -1
    assert lib.attn_merge(P, 1, 0, fake, fake, None, fake, None) == -1
    assert lib.attn_merge(P, 1, 65, fake, fake, None, fake, None) == -3
    odd = C.c_void_p(0x1004)
    assert lib.attn_merge(P, 1, 2, odd, fake, None, fake, None) == -2


def test_shard_attend_refuses_more_than_64_parts():
    lib = K.lib()
    p = K.params(4, 128, 16, 64, 512, 64, 128, 0.044)
    fake = C.c_void_p(0x1000)
    # 2^20 + 1 parts of 4096 would wrap a 32-bit product: refused before it is formed
    big = K.params(4, 128, 4096, 64, 512, 64, 128, 0.044)
    for P, n in ((p, 65), (big, (1 << 20) + 1)):
        assert lib.csa_shard_attend(C.byref(P), 1, fake, n, fake, fake, fake, fake, 1024, 0, None, 0, fake, fake,
                                    fake, fake, None, fake, 1 << 30, None) == -3
