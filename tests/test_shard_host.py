"""Host side of the sharded decode (compressed_sparse_attention_13_b200.shard)
on CPU: shard bounds, and the per-rank driver run by two gloo ranks with the
exchange over torch.distributed.  The compute phases are stand-ins written
here in float64 numpy on top of the oracle (indexer and top-k of a shard at
the shifted position t - entry0 * m, the global top-k of the gathered
candidates, a rank's partial (M, L, O), the LSE merge with the sink); the
merged result must equal the oracle's unsharded CSA and HCA attention, and
the global selection the oracle's top-k of the full scores.  This checks the
decomposition the kernels implement and the driver's exchanges (what is
gathered, in which order, which rank takes the window)."""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from compressed_sparse_attention_13_b200 import shard as SH

B, H, D, HI, DI, M_CSA, M_HCA, W, K = 2, 4, 64, 4, 32, 4, 16, 16, 48
N_CSA, N_HCA = 1000, 300


class P:
    """The parameter fields the driver reads."""
    def __init__(self, m, k):
        self.m, self.top_k, self.n_heads, self.head_dim = m, k, H, D


def _data():
    rng = np.random.default_rng(5)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return dict(q=f(B, H, D), qI=f(B, HI, DI), w=(0.1 * f(B, HI)), kv=f(B, N_CSA, D), kI=f(B, N_CSA, DI),
                kv_h=f(B, N_HCA, D), win=f(B, W, D), sinks=f(H))


def _st(a):
    return oracle.Stored(oracle.F32, np.ascontiguousarray(a, np.float32))


class NumpyOps:
    """Float64 stand-ins of the kernels' phases (see the module docstring)."""

    @staticmethod
    def select(p, batch, qI, w, sh, q_pos, device="cpu"):
        cs = np.full((batch, p.top_k), -np.inf, np.float32)
        ci = np.full((batch, p.top_k), -1, np.int32)
        for b in range(batch):
            if sh.n == 0:
                continue
            t_loc = int(q_pos[b]) - sh.entry0 * p.m
            s = oracle.indexer(_st(qI[b]), w[b][None], _st(sh.kI[b]), [t_loc], HI, p.m, W)[0]
            sel = oracle.topk(s[None].astype(np.float32), [t_loc], p.top_k, p.m, W)[0]
            ok = sel >= 0
            cs[b, ok] = s[sel[ok]]
            ci[b, ok] = sel[ok] + sh.entry0
        return torch.from_numpy(cs), torch.from_numpy(ci)

    @staticmethod
    def _partial(q, ents, win_rows, scale):
        items = np.concatenate([ents, win_rows], 0) if len(win_rows) else ents
        if items.shape[0] == 0:
            return np.zeros((H, D)), np.stack([np.full(H, -np.inf), np.zeros(H)], -1)
        lg = scale * (q.astype(np.float64) @ items.T.astype(np.float64))
        mx = lg.max(1)
        e = np.exp(lg - mx[:, None])
        return e @ items.astype(np.float64), np.stack([mx, e.sum(1)], -1)

    @staticmethod
    def _window(q_pos_b, raw_pos0_b, n_raw, raw_b):
        lo, hi = max(q_pos_b - W + 1, 0, raw_pos0_b), min(q_pos_b, raw_pos0_b + n_raw - 1)
        return raw_b[lo - raw_pos0_b: hi - raw_pos0_b + 1] if hi >= lo else raw_b[:0]

    @staticmethod
    def attend(p, batch, q, all_s, all_i, sh, raw, n_raw, raw_pos0, q_pos, idx_out, device="cpu"):
        all_s, all_i = all_s.numpy(), all_i.numpy()
        po, pml = np.zeros((batch, H, D)), np.zeros((batch, H, 2))
        for b in range(batch):
            s, ids = all_s[:, b].reshape(-1), all_i[:, b].reshape(-1)
            v = ids >= 0
            s, ids = s[v], ids[v]
            top = np.sort(ids[np.lexsort((ids, -s.astype(np.float64)))][:p.top_k])
            if idx_out is not None:
                idx_out[b] = -1
                idx_out[b, :top.size] = top
            loc = top[(top >= sh.entry0) & (top < sh.entry0 + sh.n)] - sh.entry0
            win = NumpyOps._window(int(q_pos[b]), int(raw_pos0[b]), n_raw, raw[b]) if sh.window else raw[b][:0]
            po[b], pml[b] = NumpyOps._partial(q[b], sh.kv[b][loc], win, 1 / np.sqrt(D))
        return torch.from_numpy(po), torch.from_numpy(pml)

    @staticmethod
    def hca(p, batch, q, sh, raw, n_raw, raw_pos0, q_pos, device="cpu"):
        po, pml = np.zeros((batch, H, D)), np.zeros((batch, H, 2))
        for b in range(batch):
            ne = min(max(oracle.n_elig(int(q_pos[b]), p.m, W) - sh.entry0, 0), sh.n)
            win = NumpyOps._window(int(q_pos[b]), int(raw_pos0[b]), n_raw, raw[b]) if sh.window else raw[b][:0]
            po[b], pml[b] = NumpyOps._partial(q[b], sh.kv[b][:ne], win, 1 / np.sqrt(D))
        return torch.from_numpy(po), torch.from_numpy(pml)

    @staticmethod
    def merge(p, batch, all_o, all_ml, sinks, out):
        o, ml = all_o.numpy(), all_ml.numpy()          # [parts][batch][H][..]
        Mx = np.maximum(ml[..., 0].max(0), sinks[None].astype(np.float64))
        wgt = np.where(np.isfinite(ml[..., 0]), np.exp(ml[..., 0] - Mx[None]), 0.0)
        den = (wgt * ml[..., 1]).sum(0) + np.exp(sinks[None] - Mx)
        out[:] = (wgt[..., None] * o).sum(0) / den[..., None]


def _rank(rank, world, port, res):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = _data()
        q_pos = np.array([M_CSA * N_CSA + W, 2500], np.int64)
        raw_pos0 = q_pos - W + 1
        # CSA: this rank's shard of entries and keys (per sequence)
        e0, n = SH.shard_bounds(N_CSA, world, rank)
        sh = SH.Shard(e0, n, [d["kv"][b][e0:e0 + n] for b in range(B)], [d["kI"][b][e0:e0 + n] for b in range(B)],
                      rank == world - 1)
        out = np.zeros((B, H, D))
        sel = np.zeros((B, K), np.int64)
        SH.csa_layer(P(M_CSA, K), B, d["q"], d["qI"], d["w"], sh, d["win"], W, raw_pos0, q_pos, d["sinks"], out,
                     gather=SH.nccl_gather, idx_out=sel, device="cpu", ops=NumpyOps)
        # HCA over its own entries
        qh_pos = np.array([M_HCA * N_HCA + W, 2000], np.int64)
        e0h, nh = SH.shard_bounds(N_HCA, world, rank)
        shh = SH.Shard(e0h, nh, [d["kv_h"][b][e0h:e0h + nh] for b in range(B)], None, rank == world - 1)
        out_h = np.zeros((B, H, D))
        SH.hca_layer(P(M_HCA, 1), B, d["q"], shh, d["win"], W, qh_pos - W + 1, qh_pos, d["sinks"], out_h,
                     gather=SH.nccl_gather, device="cpu", ops=NumpyOps)
        res[rank] = (out, sel, out_h, (e0, n), (e0h, nh))
    finally:
        dist.destroy_process_group()


def test_shard_bounds_cover_the_entries():
    for n_total, world in [(1000, 2), (8160, 8), (262_144, 8), (100, 4), (0, 3), (129, 1)]:
        b = [SH.shard_bounds(n_total, world, r) for r in range(world)]
        assert sum(n for _, n in b) == n_total
        assert b[0][0] == 0
        for (e0, n), (e1, _) in zip(b, b[1:]):
            assert e1 == min(e0 + n, n_total) and (n == 0 or e1 == e0 + n)
        last = max([r for r in range(world) if b[r][1]], default=-1)
        assert all(b[r][1] % 128 == 0 for r in range(last))   # all but the last non-empty shard


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_csa_and_hca_gloo_ranks_match_the_oracle(world):
    """Two ranks; and four, where the last HCA shard (the window rank) holds
    no entries: 300 entries in shards of 128, 128, 44 and 0."""
    port = 29700 + (os.getpid() * 7 + world) % 200
    with mp.get_context("spawn").Manager() as m:   # no fork of a threaded process
        res = m.dict()
        mp.start_processes(_rank, args=(world, port, res), nprocs=world, start_method="spawn")
        res = dict(res)
    assert [res[r][3] for r in range(world)] == [SH.shard_bounds(N_CSA, world, r) for r in range(world)]
    if world == 2:
        assert res[0][3] == (0, 512) and res[1][3] == (512, N_CSA - 512)
    if world == 4:
        assert [res[r][4] for r in range(world)] == [(0, 128), (128, 128), (256, 44), (300, 0)]
    d = _data()
    q_pos = np.array([M_CSA * N_CSA + W, 2500], np.int64)
    for r in range(world):                    # every rank merged the same result
        np.testing.assert_array_equal(res[r][0], res[0][0])
        np.testing.assert_array_equal(res[r][1], res[0][1])
        np.testing.assert_array_equal(res[r][2], res[0][2])
    for b in range(B):
        t = int(q_pos[b])
        s = oracle.indexer(_st(d["qI"][b]), d["w"][b][None], _st(d["kI"][b]), [t], HI, M_CSA, W)[0]
        want = oracle.topk(s[None].astype(np.float32), [t], K, M_CSA, W)[0]
        np.testing.assert_array_equal(res[0][1][b], want)
        ref = oracle.attention(_st(d["q"][b]), _st(d["kv"][b]), want[None], _st(d["win"][b]), t - W + 1,
                               d["sinks"], [t], H, M_CSA, W, 1 / np.sqrt(D))[0]
        np.testing.assert_allclose(res[0][0][b], ref, rtol=1e-9, atol=1e-12)
    qh_pos = np.array([M_HCA * N_HCA + W, 2000], np.int64)
    for b in range(B):
        t = int(qh_pos[b])
        ref = oracle.attention(_st(d["q"][b]), _st(d["kv_h"][b]), None, _st(d["win"][b]), t - W + 1, d["sinks"],
                               [t], H, M_HCA, W, 1 / np.sqrt(D))[0]
        np.testing.assert_allclose(res[0][2][b], ref, rtol=1e-9, atol=1e-12)


def _merge_by_position(cand_s, cand_i, k):
    """The selection rule of the library's candidate merge: the rank-major
    candidates of a row side by side, the k best positions by score with
    ties to the lower position, empty slots dropped, ids ascending."""
    order = np.lexsort((np.arange(cand_s.size), -cand_s.astype(np.float64)))[:k]
    ids = cand_i[order]
    return np.sort(ids[ids >= 0])


def test_merge_of_local_topk_by_position_equals_the_global_topk():
    """With heavy ties, random shard counts and eligible counts: the merge of
    the shards' local top-k (each at the shifted position t - entry0 * m)
    selects exactly the oracle's top-k of the whole row, because ranks hold
    increasing id ranges and list their candidates ascending."""
    rng = np.random.default_rng(11)
    m, W = 4, 8
    for _ in range(300):
        n = int(rng.integers(1, 400))
        k = int(rng.integers(1, 48))
        world = int(rng.integers(1, 7))
        scores = rng.integers(-3, 4, n).astype(np.float32)
        t = W + m * int(rng.integers(0, n + 3)) + int(rng.integers(0, m))
        cs, ci = [], []
        for r in range(world):
            e0, nr = SH.shard_bounds(n, world, r, align=8)
            s_loc = np.full(k, -np.inf, np.float32)
            i_loc = np.full(k, -1, np.int32)
            if nr:
                t_loc = t - e0 * m
                sel = oracle.topk(scores[e0:e0 + nr][None], [t_loc], k, m, W)[0]
                ok = sel >= 0
                s_loc[ok] = scores[e0 + sel[ok]]
                i_loc[ok] = sel[ok] + e0
            cs.append(s_loc)
            ci.append(i_loc)
        got = _merge_by_position(np.concatenate(cs), np.concatenate(ci), k)
        want = oracle.topk(scores[None], [t], k, m, W)[0]
        np.testing.assert_array_equal(got, want[want >= 0], err_msg=f"n={n} k={k} world={world} t={t}")


def test_make_shards_slices_every_sequence_and_its_scales():
    """make_shards gives rank r the rows [entry0, entry0 + n) of every
    sequence of a stored [batch][n_total] cache, codes and scales alike, as
    contiguous [batch * n] tensors; the window goes to the last rank unless
    another is named (host logic; CPU tensors)."""
    import compressed_sparse_attention_13_b200 as K
    batch, n_total, d, dI, world = 3, 700, 128, 64, 4
    g = torch.Generator().manual_seed(3)
    kv = K.empty_stored(K.FP8_S64, batch * n_total, d, device="cpu")
    kv.data.copy_(torch.randint(0, 256, kv.data.shape, generator=g, dtype=torch.uint8))
    kv.scales.copy_(torch.rand(kv.scales.shape, generator=g))
    kI = K.empty_stored(K.MXFP4, batch * n_total, dI, device="cpu")
    kI.data.copy_(torch.randint(0, 256, kI.data.shape, generator=g, dtype=torch.uint8))
    kI.scales.copy_(torch.randint(0, 256, kI.scales.shape, generator=g, dtype=torch.uint8))
    for window_rank in (None, 1):
        shards = SH.make_shards(kv, kI, batch, n_total, world, window_rank)
        assert [s.window for s in shards] == [r == (world - 1 if window_rank is None else 1) for r in range(world)]
        for r, sh in enumerate(shards):
            assert (sh.entry0, sh.n) == SH.shard_bounds(n_total, world, r)
            for st, full in ((sh.kv, kv), (sh.kI, kI)):
                assert st.fmt == full.fmt
                for part, whole in ((st.data, full.data), (st.scales, full.scales)):
                    assert part.is_contiguous() and part.shape == (batch * sh.n, whole.shape[1])
                    want = whole.reshape(batch, n_total, -1)[:, sh.entry0:sh.entry0 + sh.n].reshape(-1, whole.shape[1])
                    assert torch.equal(part, want)
    assert SH.make_shards(kv, None, batch, n_total, 2)[0].kI is None


def test_exchange_bytes():
    """A CSA step exchanges k (score, id) pairs and the partial (O and (M, L)
    per head, fp32); an HCA step the partial alone."""
    assert SH.exchange_bytes(1, 1024, 64, 512, csa=True) == 1024 * 8 + 64 * 514 * 4
    assert SH.exchange_bytes(2, 512, 8, 64, csa=False) == 2 * 8 * 66 * 4
