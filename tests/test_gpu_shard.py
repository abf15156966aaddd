"""Sharded decode (one sequence's pooled entries split over ranks along the
entry axis; "DeepSeek-V4 發佈說明", section 架構實現, and the 1M-token
context of the paper summary), with the ranks emulated one after another on
one GPU: the same C-ABI calls per rank and the same exchanged tensors
(stacked instead of all-gathered).

  * CSA: the global selection equals the unsharded csa_decode's selection
    exactly (the union of the shards' top-k contains the global top-k under
    the same order) and is valid against the oracle's scores; the merged
    output matches the oracle's attention over it (2e-2 rule and the derived
    bound).
  * HCA: the merged output matches the oracle's dense attention.
Cases: 1, 3 and 4 ranks; shards that end past a sequence's eligible entries
(a rank with nothing visible); uneven last shards; a window rank that holds
no entries; sink-dominant logits."""
import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
import oracle
import synth
from compressed_sparse_attention_13_b200 import shard as SH
from helpers import (assert_attention_close, attention_bound_stored, both_stored, check_selection, down,
                     orc_quantize, sink_dominant, up)
from synth.workloads import WORKLOADS, draw_np

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    K.csa_device_status(reset=True)
    yield
    assert K.csa_device_status(reset=True) == 0


def _bf16(bits):
    """bf16 bit patterns (as the generator draws activations) -> device tensor."""
    return up(np.ascontiguousarray(bits, np.uint16), True)


def _bf16_orc(bits):
    bits = np.ascontiguousarray(bits, np.uint16)
    return oracle.Stored(oracle.BF16, bits.reshape(-1, bits.shape[-1]))


@pytest.mark.parametrize("world,n_ctx,q_pos", [
    (1, 16384, [16384, 9000]),
    (3, 32768, [32768, 12000]),       # ranks 1-2 see few or no eligible entries of sequence 1
    (4, 32768 + 4 * 128, [33280, 20001]),  # uneven last shard
    (4, 1200, [1200, 700]),           # 300 entries: shards of 128, 128, 44 and none (the window rank)
])
def test_csa_sharded_decode_matches_unsharded_selection_and_oracle(world, n_ctx, q_pos):
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=2, n_ctx=n_ctx, seed=23)
    B, H, d, HI, dI, m, W, k = w.batch, w.H, w.d, w.HI, w.dI, w.m, w.W, w.k
    nb = w.n_blocks
    p = K.params(m, W, k, H, d, HI, dI, w.scale, K.BF16, K.FP8_S64, K.MXFP4)
    kv_h, kI_h, qI_h = draw_np(w, "kv"), draw_np(w, "kI"), draw_np(w, "qI")
    kv_d, _ = both_stored(kv_h.reshape(-1, d), "fp8")
    kI_d, _ = both_stored(kI_h.reshape(-1, dI), "mxfp4")
    qI_d, _ = both_stored(qI_h.reshape(-1, dI), "mxfp4")
    q_h, win_h, wt, sinks = draw_np(w, "q"), draw_np(w, "window"), draw_np(w, "w"), draw_np(w, "sinks")
    q, win = _bf16(q_h), _bf16(win_h)
    q_pos = np.asarray(q_pos, np.int64)
    raw_pos0 = q_pos - W + 1
    shards = SH.make_shards(kv_d, kI_d, B, nb, world)
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, k, dtype=torch.int32, device="cuda")
    SH.emulate_csa_layer(p, B, q, qI_d, up(wt), shards, win, W, up(raw_pos0), up(q_pos), up(sinks), out,
                         idx_out=sel)
    # the unsharded decode of the same inputs
    out1 = torch.empty_like(out)
    sel1 = torch.empty_like(sel)
    ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, B, 1, nb), dtype=torch.uint8, device="cuda")
    K.csa_decode(p, B, q, qI_d, up(wt), kv_d, kI_d, nb, win, W, up(raw_pos0), up(q_pos), up(sinks), out1, sel1,
                 ws)
    torch.cuda.synchronize()
    got, got_sel = down(out.float()), down(sel)
    assert np.array_equal(got_sel, down(sel1)), "sharded selection differs from the unsharded one"
    for b in range(B):
        t = int(q_pos[b])
        qI_o, kI_o = orc_quantize(qI_h[b].reshape(-1, dI), "mxfp4"), orc_quantize(kI_h[b], "mxfp4")
        scores = oracle.indexer(qI_o, wt[b][None], kI_o, [t], HI, m, W)[0]
        check_selection(got_sel[b], scores, min(oracle.n_elig(t, m, W), nb), k, what=f"seq {b}")
        args = (_bf16_orc(q_h[b]), orc_quantize(kv_h[b], "fp8"), got_sel[b][None], _bf16_orc(win_h[b]), t - W + 1)
        ref = oracle.attention(*args, sinks, [t], H, m, W, w.scale)[0]
        bound = attention_bound_stored(*args, sinks, [t], H, m, W, w.scale)[0]
        assert_attention_close(got[b], ref, bound, f"sharded seq {b}")


@pytest.mark.parametrize("world,sink_shift", [(4, None), (3, 2.0), (8, None)])
def test_hca_sharded_decode_matches_oracle(world, sink_shift):
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=2, n_ctx=1 << 20, m=128, seed=29)
    B, H, d, m, W = w.batch, w.H, w.d, w.m, w.W
    nb = w.n_blocks                     # 8192 entries of 128 tokens
    p = K.params(m, W, 1, H, d, 1, 32, w.scale, K.BF16, K.FP8_S64, K.MXFP4)
    kv_h = draw_np(w, "kv")
    kv_d, _ = both_stored(kv_h.reshape(-1, d), "fp8")
    q_h, win_h, sinks = draw_np(w, "q"), draw_np(w, "window"), draw_np(w, "sinks")
    q_pos = np.array([1 << 20, 300_000], np.int64)   # sequence 1 sees 2,342 entries: later ranks none
    raw_pos0 = q_pos - W + 1
    kv_o = [orc_quantize(kv_h[b], "fp8") for b in range(B)]
    if sink_shift is not None:
        sinks = np.max([sink_dominant(_bf16_orc(q_h[b]), kv_o[b], None, _bf16_orc(win_h[b]), int(raw_pos0[b]),
                                      [int(q_pos[b])], H, m, W, w.scale, sink_shift) for b in range(B)], axis=0)
    shards = SH.make_shards(kv_d, None, B, nb, world)
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    SH.emulate_hca_layer(p, B, _bf16(q_h), shards, _bf16(win_h), W, up(raw_pos0), up(q_pos), up(sinks), out)
    torch.cuda.synchronize()
    got = down(out.float())
    for b in range(B):
        t = int(q_pos[b])
        args = (_bf16_orc(q_h[b]), kv_o[b], None, _bf16_orc(win_h[b]), t - W + 1)
        ref = oracle.attention(*args, sinks, [t], H, m, W, w.scale)[0]
        bound = attention_bound_stored(*args, sinks, [t], H, m, W, w.scale)[0]
        assert_attention_close(got[b], ref, bound, f"hca sharded seq {b}")


def test_attn_merge_of_one_part_is_the_normalised_partial():
    """attn_merge over a single partial with no sink divides O by L (the
    partial from hca_shard_attend of the whole cache, no window)."""
    w = WORKLOADS["csa_decode_128k_b32"].with_(batch=1, n_ctx=65536, m=128, seed=31)
    B, H, d, m, W = w.batch, w.H, w.d, w.m, w.W
    nb = w.n_blocks
    p = K.params(m, W, 1, H, d, 1, 32, w.scale, K.BF16, K.FP8_S64, K.MXFP4)
    kv_h = draw_np(w, "kv")
    kv_d, _ = both_stored(kv_h.reshape(-1, d), "fp8")
    q_h = draw_np(w, "q")
    q_pos = np.array([65536], np.int64)
    sh = SH.Shard(0, nb, kv_d, None, False)
    po, pml = SH.hca_attend(p, B, _bf16(q_h), sh, None, 0, up(q_pos - W + 1), up(q_pos))
    out = torch.empty(B, H, d, dtype=torch.bfloat16, device="cuda")
    K.attn_merge(p, B, 1, po[None].contiguous(), pml[None].contiguous(), None, out)
    torch.cuda.synchronize()
    ml = down(pml)
    assert np.all(np.isfinite(ml[..., 0])) and np.all(ml[..., 1] >= 1.0)   # the max item contributes e^0
    ref = down(po) / ml[..., 1:2]
    got = down(out.float())
    assert np.max(np.abs(got - ref)) <= 2 ** -8 * np.max(np.abs(ref)) + 1e-6
    # and the oracle's dense attention over the same entries without window or sink
    n_e = oracle.n_elig(65536, m, W)
    args = (_bf16_orc(q_h[0]), orc_quantize(kv_h[0][:n_e], "fp8"), None,
            oracle.Stored(oracle.BF16, np.zeros((0, d), np.uint16)), 65536 - W + 1)
    ref_o = oracle.attention(*args, None, [65536], H, m, W, w.scale)[0]
    bound = attention_bound_stored(*args, None, [65536], H, m, W, w.scale)[0]
    assert_attention_close(got[0], ref_o, bound, "one-part merge")


@pytest.mark.parametrize("world", [2, 3])
def test_fp32_sharded_decode_matches_oracle_to_1e5(world):
    """The fp32 formats (CUDA-core indexer and attention, fp32 entries) through
    the sharded CSA and HCA paths: the merged outputs match the oracle's
    unsharded attention within 1e-5, which pins the partial (M, L, O) and the
    LSE merge arithmetic tightly; the selection is valid against the oracle's
    scores."""
    from helpers import assert_close_f32
    B, H, d, HI, dI, m, W, k = 2, 8, 64, 4, 32, 4, 64, 16
    rng_seed = 61
    nb = 1024
    st = lambda a: oracle.Stored(oracle.F32, np.ascontiguousarray(a, np.float32).reshape(-1, a.shape[-1]))
    q_h = synth.tensor_np(rng_seed, "f32s/q", (B, H, d))
    qI_h = synth.tensor_np(rng_seed, "f32s/qI", (B, HI, dI))
    w_h = synth.tensor_np(rng_seed, "f32s/w", (B, HI), std=0.1)
    kv_h = synth.tensor_np(rng_seed, "f32s/kv", (B, nb, d))
    kI_h = synth.tensor_np(rng_seed, "f32s/kI", (B, nb, dI))
    win_h = synth.tensor_np(rng_seed, "f32s/win", (B, W, d))
    sinks = synth.tensor_np(rng_seed, "f32s/sinks", (H,))
    q_pos = np.array([m * nb + W, m * 300 + W + 3], np.int64)
    raw_pos0 = q_pos - W + 1
    p = K.params(m, W, k, H, d, HI, dI, 1 / 8, K.F32, K.F32, K.F32)
    kv_d = K.Stored(K.F32, up(kv_h.reshape(-1, d)))
    kI_d = K.Stored(K.F32, up(kI_h.reshape(-1, dI)))
    shards = SH.make_shards(kv_d, kI_d, B, nb, world)
    out = torch.empty(B, H, d, dtype=torch.float32, device="cuda")
    sel = torch.empty(B, k, dtype=torch.int32, device="cuda")
    SH.emulate_csa_layer(p, B, up(q_h), K.Stored(K.F32, up(qI_h.reshape(-1, dI))), up(w_h), shards, up(win_h), W,
                         up(raw_pos0), up(q_pos), up(sinks), out, idx_out=sel)
    torch.cuda.synchronize()
    got, got_sel = down(out), down(sel)
    for b in range(B):
        t = int(q_pos[b])
        scores = oracle.indexer(st(qI_h[b]), w_h[b][None], st(kI_h[b]), [t], HI, m, W)[0]
        check_selection(got_sel[b], scores, min(oracle.n_elig(t, m, W), nb), k, what=f"fp32 seq {b}")
        ref = oracle.attention(st(q_h[b]), st(kv_h[b]), got_sel[b][None], st(win_h[b]), t - W + 1, sinks, [t], H, m,
                               W, 1 / 8)[0]
        assert_close_f32(got[b], ref, 1e-5, f"fp32 sharded csa seq {b}")
    # HCA at m' = 16 over the same entries
    ph = K.params(16, W, 1, H, d, 1, 32, 1 / 8, K.F32, K.F32, K.F32)
    qh_pos = np.array([16 * nb + W, 16 * 200 + W + 5], np.int64)
    hsh = SH.make_shards(kv_d, None, B, nb, world)
    SH.emulate_hca_layer(ph, B, up(q_h), hsh, up(win_h), W, up(qh_pos - W + 1), up(qh_pos), up(sinks), out)
    torch.cuda.synchronize()
    got = down(out)
    for b in range(B):
        t = int(qh_pos[b])
        ref = oracle.attention(st(q_h[b]), st(kv_h[b]), None, st(win_h[b]), t - W + 1, sinks, [t], H, 16, W, 1 / 8)[0]
        assert_close_f32(got[b], ref, 1e-5, f"fp32 sharded hca seq {b}")
