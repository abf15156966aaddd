"""Pins for the oracle's number formats and quantisers.

Each check ties the oracle to something other than itself: the OCP spec tables
(golden fixtures), torch's own float8_e4m3fn cast (a library routine), or brute
force over every code.
"""
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines


def test_e2m1_table_matches_ocp_spec(orc):
    for code, val in golden_lines("e2m1_table.txt"):
        v = orc.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_points_match_ofp8_spec(orc):
    for code, val in golden_lines("e4m3_points.txt"):
        v = orc.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(v)
        else:
            assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_exhaustive_against_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e8m0_and_bf16(orc):
    assert orc.e8m0_value(127) == 1.0
    assert orc.e8m0_value(0) == 2.0 ** -127
    assert orc.e8m0_value(254) == 2.0 ** 127
    assert math.isnan(orc.e8m0_value(255))
    for bits in (0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F):
        ref = torch.tensor([bits], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
        assert orc.bf16_value(bits) == ref.double().item()


def _e4m3_brute(q):
    """Nearest finite E4M3 code to each value, ties to even code, saturating."""
    vals = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    vals = vals.double().numpy()
    pos = np.arange(0, 0x7F)  # finite non-negative codes 0x00..0x7E
    out = np.empty(q.shape, dtype=np.uint8)
    for i, x in enumerate(q.reshape(-1)):
        a = min(abs(float(x)), 448.0)
        dist = np.abs(vals[pos] - a)
        best = pos[dist == dist.min()]
        c = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        if math.copysign(1, float(x)) < 0:
            c |= 0x80
        out.reshape(-1)[i] = c
    return out


def test_fp8_quantiser_against_brute_force_and_torch(orc):
    rng = np.random.default_rng(0)
    v = rng.standard_normal((6, 128)).astype(np.float32)
    v[1] *= 1e-3
    v[2, :64] = 0.0                       # all-zero group -> scale 1, codes 0
    v[3, 5] = 1e4                         # one large value dominates its group
    v[4] = np.float32(448.0)              # exact grid values survive
    st = orc.quantize_fp8_s64(v)
    assert st.scales.shape == (6, 2) and st.data.shape == (6, 128)
    amax = np.abs(v.reshape(6, 2, 64)).max(-1)
    exp_scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(st.scales, exp_scale)
    q = (v.reshape(6, 2, 64) / st.scales[:, :, None]).astype(np.float32).reshape(6, 128)
    assert np.array_equal(st.data, _e4m3_brute(q))
    # torch's cast is round-to-nearest-even too (it gives NaN instead of
    # saturating, which never happens here since |q| <= 448)
    tq = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(st.data, tq)
    deq = orc.dequantize(st)
    assert np.all(np.abs(deq - v) <= np.repeat(st.scales, 64, axis=1) * 16 + 1e-30)


def _e2m1_brute(a):
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    a = min(a, 6.0)
    d = np.abs(grid - a)
    best = np.flatnonzero(d == d.min())
    return int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])


def test_mxfp4_quantiser_against_brute_force(orc):
    rng = np.random.default_rng(1)
    v = rng.standard_normal((5, 64)).astype(np.float32)
    v[1, :32] = 0.0                                   # zero block -> X = 0
    v[2] *= 100.0
    v[3, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 4, np.float32)  # ties
    v[4, :32] *= 2.0 ** -20
    st = orc.quantize_mxfp4(v)
    assert st.data.shape == (5, 32) and st.scales.shape == (5, 2)
    for r in range(5):
        for g in range(2):
            blk = v[r, 32 * g:32 * g + 32].astype(np.float64)
            amax = np.abs(blk).max()
            X = 0 if amax == 0 else math.floor(math.log2(amax)) - 2
            assert st.scales[r, g] == X + 127
            for i in range(32):
                col = 32 * g + i
                byte = st.data[r, col // 2]
                code = (byte >> 4) if col & 1 else (byte & 15)
                exp = _e2m1_brute(abs(blk[i]) / 2.0 ** X) | (8 if blk[i] < 0 or
                                                             math.copysign(1, blk[i]) < 0 else 0)
                assert code == exp, (r, g, i, blk[i], code, exp)
    # the tie row: 0.25->0, 0.75->1.0, 1.25->1.0, 1.75->2, 2.5->2, 3.5->4, 5->4, 6->6 at X=0
    deq = orc.dequantize(st)
    assert st.scales[3, 0] == 127
    assert list(deq[3, :8]) == [0, 1, 1, 2, 2, 4, 4, 6]


def test_every_code_round_trips(orc):
    # decode(code) * scale quantises back to the same code (no double rounding)
    for code in range(256):
        if code in (0x7F, 0xFF):
            continue
        v = np.zeros((1, 64), np.float32)
        v[0, 0] = 448.0                    # pins scale = 1
        v[0, 1] = orc.e4m3_value(code)
        st = orc.quantize_fp8_s64(v)
        assert st.scales[0, 0] == 1.0
        got = st.data[0, 1]
        assert got == code or (orc.e4m3_value(code) == 0 and orc.e4m3_value(got) == 0)
    for code in range(16):
        v = np.zeros((1, 32), np.float32)
        v[0, 0] = 6.0                      # pins X = 0
        v[0, 1] = orc.e2m1_value(code)
        st = orc.quantize_mxfp4(v)
        c = st.data[0, 0] >> 4
        assert c == code or (orc.e2m1_value(code) == 0 and orc.e2m1_value(c) == 0)


@pytest.mark.parametrize("n", [1, 7, 1000])
def test_bf16_storage_rounding_matches_torch(orc, n):
    v = np.random.default_rng(n).standard_normal(n).astype(np.float32) * 3
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.f32_to_bf16(v), ref)
