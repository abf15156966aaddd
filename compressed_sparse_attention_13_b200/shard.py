"""Sharded decode of long sequences: the pooled entries of every sequence are
split over ranks along the entry axis (one process per GPU), with one
exchange per step of the method ("DeepSeek-V4 發佈說明", section 架構實現 and
the paper summary's 1M-token context).

Rank r holds the contiguous entries [entry0, entry0 + n) of each sequence.
A CSA layer is

    csa_shard_select   (every rank: indexer + local top-k -> k candidates)
    all-gather         (candidates, rank-major [world][batch][k])
    csa_shard_attend   (every rank: exact global top-k, partial attention
                        over the selected entries it holds, and the window on
                        the window rank)
    all-gather         (partials, rank-major)
    attn_merge         (LSE merge with the sink -> the layer output)

and an HCA layer is hca_shard_attend, all-gather, attn_merge.  All arithmetic
runs in the library's kernels; this module only sizes buffers, calls the
C-ABI and hands tensors to the exchange.  The exchange is a callable
`gather(t) -> [world, *t.shape]`: `nccl_gather` (torch.distributed; NCCL
over NVLink on GPUs) for real ranks, or a stacking of per-rank tensors when
the ranks are emulated one after another on one device (`emulate_*`)."""
from __future__ import annotations

from dataclasses import dataclass

import compressed_sparse_attention_13_b200 as K


def shard_bounds(n_total: int, world: int, rank: int, align: int = 128):
    """(entry0, n) of `rank`: equal contiguous shards whose sizes are
    multiples of `align` (the indexer's key step), the last one shorter."""
    per = -(-n_total // world)
    per = -(-per // align) * align
    entry0 = min(rank * per, n_total)
    return entry0, max(0, min(per, n_total - entry0))


def nccl_gather(t):
    """All-gather over the default process group, rank-major
    [world, *t.shape]: one collective into one buffer (flattened, so every
    backend splits it by rank the same way), with no per-rank copies."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size()
    out = torch.empty(world * t.numel(), dtype=t.dtype, device=t.device)
    dist.all_gather_into_tensor(out, t.contiguous().reshape(-1))
    return out.view((world,) + tuple(t.shape))


@dataclass
class Shard:
    """One rank's view of the layer: its entries (and indexer keys) and
    whether it attends to the raw window."""
    entry0: int
    n: int
    kv: "K.Stored"
    kI: "K.Stored | None" = None
    window: bool = False


def _ws(p, op, batch, n, device):
    import torch
    return torch.empty(K.csa_workspace_size(p, op, batch, 1, max(n, 0)), dtype=torch.uint8, device=device)


def csa_select(p, batch, qI, w, sh: Shard, q_pos, device="cuda"):
    """Phase 1 of a CSA layer on one rank: (cand_scores, cand_ids) [batch][k]."""
    import torch
    cs = torch.empty(batch, p.top_k, dtype=torch.float32, device=device)
    ci = torch.empty(batch, p.top_k, dtype=torch.int32, device=device)
    K.csa_shard_select(p, batch, qI, w, sh.kI, sh.n, sh.entry0, q_pos, cs, ci,
                       _ws(p, K.OP_SHARD_SELECT, batch, sh.n, device))
    return cs, ci


def _partials(p, batch, device):
    import torch
    return (torch.empty(batch, p.n_heads, p.head_dim, dtype=torch.float32, device=device),
            torch.empty(batch, p.n_heads, 2, dtype=torch.float32, device=device))


def csa_attend(p, batch, q, all_scores, all_ids, sh: Shard, raw, n_raw, raw_pos0, q_pos, idx_out=None,
               device="cuda"):
    """Phase 2 of a CSA layer on one rank: this rank's partial (O, (M, L))."""
    po, pml = _partials(p, batch, device)
    n_parts = all_scores.shape[0]
    K.csa_shard_attend(p, batch, q, n_parts, all_scores, all_ids, sh.kv, sh.n, sh.entry0,
                       raw if sh.window else None, n_raw if sh.window else 0, raw_pos0, q_pos, po, pml,
                       idx_out, _ws(p, K.OP_SHARD_ATTEND, batch, sh.n, device))
    return po, pml


def hca_attend(p, batch, q, sh: Shard, raw, n_raw, raw_pos0, q_pos, device="cuda"):
    """An HCA layer's partial on one rank."""
    po, pml = _partials(p, batch, device)
    K.hca_shard_attend(p, batch, q, sh.kv, sh.n, sh.entry0, raw if sh.window else None,
                       n_raw if sh.window else 0, raw_pos0, q_pos, po, pml,
                       _ws(p, K.OP_HCA_SHARD, batch, sh.n, device))
    return po, pml


def merge(p, batch, all_o, all_ml, sinks, out):
    K.attn_merge(p, batch, all_o.shape[0], all_o, all_ml, sinks, out)


class LibraryOps:
    """The phases as the library's kernels run them."""
    select = staticmethod(csa_select)
    attend = staticmethod(csa_attend)
    hca = staticmethod(hca_attend)
    merge = staticmethod(merge)


# ------------------------------------------------------------ one rank's step
def csa_layer(p, batch, q, qI, w, sh: Shard, raw, n_raw, raw_pos0, q_pos, sinks, out, gather=nccl_gather,
              idx_out=None, device="cuda", ops=LibraryOps):
    """One CSA layer decode step as one rank of the group `gather` spans;
    every rank takes the same two exchanges in the same order."""
    cs, ci = ops.select(p, batch, qI, w, sh, q_pos, device=device)
    all_s, all_i = gather(cs), gather(ci)
    po, pml = ops.attend(p, batch, q, all_s, all_i, sh, raw, n_raw, raw_pos0, q_pos, idx_out, device=device)
    ops.merge(p, batch, gather(po), gather(pml), sinks, out)


def hca_layer(p, batch, q, sh: Shard, raw, n_raw, raw_pos0, q_pos, sinks, out, gather=nccl_gather,
              device="cuda", ops=LibraryOps):
    """One HCA layer decode step as one rank of the group `gather` spans."""
    po, pml = ops.hca(p, batch, q, sh, raw, n_raw, raw_pos0, q_pos, device=device)
    ops.merge(p, batch, gather(po), gather(pml), sinks, out)


# ------------------------------------------- every rank in turn on one device
def emulate_csa_layer(p, batch, q, qI, w, shards, raw, n_raw, raw_pos0, q_pos, sinks, out, idx_out=None,
                      device="cuda"):
    """The CSA layer of len(shards) ranks run one after another on one device
    (each rank's phase, then the stacked exchange): the same calls and data
    movement as csa_layer on every rank, for testing and for timing a rank's
    share of the work."""
    import torch
    cand = [csa_select(p, batch, qI, w, sh, q_pos, device) for sh in shards]
    all_s = torch.stack([c[0] for c in cand])
    all_i = torch.stack([c[1] for c in cand])
    parts = [csa_attend(p, batch, q, all_s, all_i, sh, raw, n_raw, raw_pos0, q_pos,
                        idx_out if r == 0 else None, device) for r, sh in enumerate(shards)]
    merge(p, batch, torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]), sinks, out)


def emulate_hca_layer(p, batch, q, shards, raw, n_raw, raw_pos0, q_pos, sinks, out, device="cuda"):
    import torch
    parts = [hca_attend(p, batch, q, sh, raw, n_raw, raw_pos0, q_pos, device) for sh in shards]
    merge(p, batch, torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]), sinks, out)


def split_entries(st: "K.Stored", batch: int, n_total: int, entry0: int, n: int):
    """The [batch][n] slice of a stored [batch][n_total][...] tensor (as a
    contiguous copy: a rank's own memory)."""
    def part(t):
        if t is None:
            return None
        width = t.numel() // max(1, batch * n_total)
        v = t.reshape(batch, n_total, width)[:, entry0:entry0 + n]
        return v.contiguous().reshape(batch * n, width)
    return K.Stored(st.fmt, part(st.data), part(st.scales))


def make_shards(kv, kI, batch, n_total, world, window_rank=None):
    """Split stored entries (and keys) into `world` shards; the last rank
    attends to the window unless another is named."""
    window_rank = world - 1 if window_rank is None else window_rank
    out = []
    for r in range(world):
        e0, n = shard_bounds(n_total, world, r)
        out.append(Shard(e0, n, split_entries(kv, batch, n_total, e0, n),
                         None if kI is None else split_entries(kI, batch, n_total, e0, n), r == window_rank))
    return out


def exchange_bytes(batch: int, k: int, H: int, d: int, csa: bool = True) -> int:
    """Bytes one rank contributes to the exchanges of a decode step: the k
    candidates (score + id) of a CSA layer, then the partial (O and (M, L)
    per head)."""
    return (batch * k * 8 if csa else 0) + batch * H * (d + 2) * 4


__all__ = ["Shard", "LibraryOps", "shard_bounds", "nccl_gather", "csa_select", "csa_attend", "hca_attend",
           "merge", "csa_layer", "hca_layer", "emulate_csa_layer", "emulate_hca_layer", "split_entries",
           "make_shards", "exchange_bytes"]
