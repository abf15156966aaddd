"""csa_decode_noalloc: the same decode step as csa_decode, computed on the
library's fixed device scratch instead of a caller workspace.  Two calls in a
row on different inputs must each give exactly what csa_decode gives on the
same inputs (same kernels, same arithmetic: bitwise equal), and a request
larger than the scratch is refused on the host."""
import ctypes as C

import numpy as np
import pytest
import torch

import compressed_sparse_attention_13_b200 as K
from helpers import FMT, act_dev, both_stored, down, up
from synth.workloads import WORKLOADS, draw_np


def test_oversize_request_is_refused_on_the_host():
    """Refused before the device is touched, so this runs without a GPU."""
    p = K.params(4, 128, 512, 64, 512, 64, 128, 0.044)
    batch, max_blocks = 256, 1 << 16
    assert K.csa_workspace_size(p, K.OP_DECODE, batch, 1, max_blocks) > K.NOALLOC_SCRATCH_BYTES
    st = K.lib().csa_decode_noalloc(C.byref(p), batch, *([None] * 8), max_blocks, None, 128,
                                    None, None, None, None, None, None)
    assert st == K.ERR_WORKSPACE


def _decode_inputs(w):
    B, d, dI, W = w.batch, w.d, w.dI, w.W
    q, qI, wt = draw_np(w, "q"), draw_np(w, "qI"), draw_np(w, "w")
    kv, kI, win, sinks = draw_np(w, "kv"), draw_np(w, "kI"), draw_np(w, "window"), draw_np(w, "sinks")
    kv_d, _ = both_stored(kv.reshape(-1, d), w.kv)
    kI_d, _ = both_stored(kI.reshape(-1, dI), w.idx)
    qI_d, _ = both_stored(qI.reshape(-1, dI), w.idx)
    rng = np.random.default_rng(w.seed)
    q_pos = np.sort(rng.integers(W + 1, w.n_ctx + 1, size=B)).astype(np.int64)
    q_pos[-1] = w.n_ctx
    return dict(q=act_dev(q, w.act), qI=qI_d, w=up(wt), kv=kv_d, kI=kI_d,
                raw=act_dev(win, w.act), raw_pos0=up(q_pos - W + 1), q_pos=up(q_pos),
                sinks=up(sinks))


@pytest.mark.gpu
def test_noalloc_matches_csa_decode_on_two_calls_in_a_row():
    K.csa_device_status(reset=True)
    base = WORKLOADS["csa_decode_128k_b32"].with_(batch=6, n_ctx=20000)
    p = K.params(base.m, base.W, base.k, base.H, base.d, base.HI, base.dI, base.scale,
                 FMT[base.act], FMT[base.kv], FMT[base.idx])
    nb = base.n_blocks
    assert K.csa_workspace_size(p, K.OP_DECODE, base.batch, 1, nb) <= K.NOALLOC_SCRATCH_BYTES
    for seed in (21, 22):
        w = base.with_(seed=seed)
        a = _decode_inputs(w)
        shape = (w.batch, w.H, w.d)
        ref_out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
        ref_sel = torch.empty((w.batch, w.k), dtype=torch.int32, device="cuda")
        ws = torch.empty(K.csa_workspace_size(p, K.OP_DECODE, w.batch, 1, nb), dtype=torch.uint8,
                         device="cuda")
        K.csa_decode(p, w.batch, a["q"], a["qI"], a["w"], a["kv"], a["kI"], nb, a["raw"], w.W,
                     a["raw_pos0"], a["q_pos"], a["sinks"], ref_out, ref_sel, ws)
        out = torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda")
        sel = torch.full((w.batch, w.k), -7, dtype=torch.int32, device="cuda")
        K.csa_decode_noalloc(p, w.batch, a["q"], a["qI"], a["w"], a["kv"], a["kI"], nb, a["raw"],
                             w.W, a["raw_pos0"], a["q_pos"], a["sinks"], out, sel)
        got_sel, want_sel = down(sel), down(ref_sel)
        assert np.array_equal(got_sel, want_sel), f"seed {seed}: selections differ"
        # the same kernels on the same inputs: the outputs are bitwise equal
        got, want = down(out), down(ref_out)
        assert np.array_equal(got, want), f"seed {seed}: outputs differ"
        assert K.csa_device_status(reset=True) == 0
