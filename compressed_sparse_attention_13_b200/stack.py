"""Interleaved CSA / HCA layers with incremental pooling ("DeepSeek-V4 發佈說明",
section 架構實現: CSA and HCA layers interleave; new tokens enter the sliding
window and every completed block of m (CSA) or m' (HCA) tokens is pooled into
one more compressed entry).

A driver over the C-ABI entry points: it owns the per-layer caches (torch
allocations) and calls csa_compress / csa_prefill / csa_decode / hca_attn in
order.  No arithmetic of the method happens here.  One sequence per layer
(batch 1): the raw-token buffer is a single linear window whose first row is
at position `raw_pos0`.

Per token t of a layer the caller supplies its raw value x_t and gate logits
z_t (act format, [d]); CSA layers also take the indexer-key inputs xI_t, zI_t
([dI]), which are pooled the same way (d = dI) and stored as MXFP4 keys.
"""
from __future__ import annotations

from dataclasses import dataclass

from . import (BF16, FP8_S64, MXFP4, OP_DECODE, OP_HCA_ATTN, OP_PREFILL, OP_WINDOW_ATTN, Params,
               csa_compress, csa_decode, csa_prefill, csa_workspace_size, empty_stored, hca_attn,
               window_attn)


def v4_pro_schedule(n_layers: int = 61, mtp: bool = True) -> list:
    """Attention kind of each layer of DeepSeek-V4-Pro ("DeepSeek-V4 發佈說明",
    section 架構實現: 61 layers; layers 0-1 use HCA, layers 2-60 alternate
    between CSA and HCA, and the final MTP block uses only sliding-window
    attention).  The alternation is read as starting with CSA at layer 2, the
    order the note names them in; the MTP block is appended as a 62nd entry."""
    kinds = ["hca" if i < 2 else ("csa" if (i - 2) % 2 == 0 else "hca") for i in range(n_layers)]
    return kinds + (["window"] if mtp else [])


@dataclass
class LayerSpec:
    kind: str          # "csa" | "hca" | "window" (the MTP block: sliding window only)
    p: Params          # m, window, top_k, heads, dims, scale, formats
    prior_tokens: int  # tokens already pooled into the cache (a multiple of m)
    new_tokens: int    # capacity for tokens appended after the prior cache


class Layer:
    """Caches of one layer.  kv / kI rows [0, prior_tokens / m) are filled by
    the caller (see `kv`, `kI`); later rows are pooled here as blocks complete."""

    def __init__(self, spec: LayerSpec, device="cuda"):
        import torch
        self.spec = spec
        p = spec.p
        self.m, self.W, self.d = p.m, p.window, p.head_dim
        # capacity in whole 128-row steps: the tensor-core MXFP4 indexer takes
        # a row count that is a multiple of 4 (rows past the pooled ones are
        # never read: only n_elig(t) entries are visible)
        self.cap_blocks = -(-((spec.prior_tokens + spec.new_tokens) // self.m) // 128) * 128
        # the window-only block keeps no pooled cache
        self.kv = empty_stored(FP8_S64, self.cap_blocks, self.d, device) if spec.kind != "window" else None
        self.kI = empty_stored(MXFP4, self.cap_blocks, p.idx_dim, device) if spec.kind == "csa" else None
        # raw window: the W - 1 tokens before the first new token, then the new tokens
        self.raw_pos0 = spec.prior_tokens - (self.W - 1) if self.W > 0 else spec.prior_tokens
        self.n_raw = max(self.W - 1, 0) + spec.new_tokens
        dt = torch.bfloat16
        self.x = torch.zeros(self.n_raw, self.d, dtype=dt, device=device)
        self.z = torch.zeros(self.n_raw, self.d, dtype=dt, device=device)
        if spec.kind == "csa":
            self.xI = torch.zeros(self.n_raw, p.idx_dim, dtype=dt, device=device)
            self.zI = torch.zeros(self.n_raw, p.idx_dim, dtype=dt, device=device)
        self.pos0 = torch.tensor([self.raw_pos0], dtype=torch.int64, device=device)
        self.t_next = spec.prior_tokens  # position of the next new token
        self._pooled = (spec.prior_tokens + self.m - 1) // self.m
        # decode workspace, allocated once so that decode steps can be captured in a graph
        op = {"csa": OP_DECODE, "hca": OP_HCA_ATTN, "window": OP_WINDOW_ATTN}[spec.kind]
        self.ws = torch.empty(csa_workspace_size(p, op, 1, 1, self.cap_blocks), dtype=torch.uint8,
                              device=device)

    def _row(self, t):
        return t - self.raw_pos0

    def _pool_completed(self, t_end, bias, biasI):
        """Pool every block that completes at or before position t_end - 1 and
        has not been pooled yet."""
        if self.kv is None:
            return
        m, d = self.m, self.d
        for j in range(self._pooled, t_end // m):
            r0 = self._row(j * m)
            csa_compress(self.spec.p, d, self.x[r0:r0 + m], self.z[r0:r0 + m], bias, m,
                         _rows(self.kv, j))
            if self.kI is not None:
                csa_compress(self.spec.p, self.spec.p.idx_dim, self.xI[r0:r0 + m],
                             self.zI[r0:r0 + m], biasI, m, _rows(self.kI, j))
            self._pooled = j + 1

    def set_prior_window(self, x_prior):
        """Raw values of the W - 1 tokens before the first new token (they are
        already pooled; only the window branch reads them)."""
        n = self.W - 1
        if n > 0:
            self.x[:n].copy_(x_prior[-n:])

    def append(self, x, z, xI=None, zI=None):
        """Write the raw inputs of the next len(x) tokens into the window."""
        n = x.shape[0]
        r = self._row(self.t_next)
        self.x[r:r + n].copy_(x)
        self.z[r:r + n].copy_(z)
        if self.kI is not None:
            self.xI[r:r + n].copy_(xI)
            self.zI[r:r + n].copy_(zI)
        self.t_next += n

    def decode(self, q, qI, w, sinks, out, idx_out, bias, biasI=None, q_pos=None):
        """Attention of the newest token (already appended), then pooling of a
        block it completes.  q_pos: a device int64 [1] holding the token's
        position (made here when not given; pass one to capture steps in a graph)."""
        import torch
        spec, p = self.spec, self.spec.p
        t = self.t_next - 1
        if q_pos is None:
            q_pos = torch.tensor([t], dtype=torch.int64, device=q.device)
        if spec.kind == "csa":
            csa_decode(p, 1, q, qI, w, self.kv, self.kI, self.cap_blocks, self.x, self.n_raw,
                       self.pos0, q_pos, sinks, out, idx_out, self.ws)
        elif spec.kind == "hca":
            hca_attn(p, 1, 1, q, self.kv, self.cap_blocks, self.x, self.n_raw, self.pos0, q_pos,
                     sinks, out, self.ws)
        else:
            window_attn(p, 1, 1, q, self.x, self.n_raw, self.pos0, q_pos, sinks, out, self.ws)
        self._pool_completed(t + 1, bias, biasI)

    def state(self):
        """(next position, blocks pooled): with restore(), replays the same steps."""
        return self.t_next, self._pooled

    def restore(self, st):
        self.t_next, self._pooled = st

    def prefill(self, T, q, qI, w, sinks, out, idx_out, bias, biasI=None):
        """A chunk of the T newest tokens (already appended, starting at a
        multiple of m): pool its blocks, then attend every chunk query."""
        import torch
        spec, p = self.spec, self.spec.p
        t0 = self.t_next - T
        assert t0 % self.m == 0 and t0 == spec.prior_tokens, "one chunk, right after the prior cache"
        r0 = self._row(t0)
        # only the chunk's complete blocks are pooled now; a partial last block
        # is pooled by the decode step that completes it
        nb = T // self.m
        n_pool = nb * self.m
        if spec.kind == "csa":
            # indexer keys of the chunk's blocks first: csa_prefill reads them
            csa_compress(p, p.idx_dim, self.xI[r0:r0 + n_pool], self.zI[r0:r0 + n_pool], biasI,
                         n_pool, _rows(self.kI, t0 // self.m, nb))
            ws = torch.empty(csa_workspace_size(p, OP_PREFILL, 1, T, self.cap_blocks),
                             dtype=torch.uint8, device=q.device)
            # first raw row the chunk's windows need (the chunk itself when W = 0)
            rp0 = t0 - (self.W - 1) if self.W > 0 else t0
            rs = self._row(rp0)
            csa_prefill(p, 1, T, t0, self.x[rs:], self.n_raw - rs, rp0, self.z[r0:r0 + T],
                        bias, q, qI, w, self.kv, self.kI, self.cap_blocks, sinks, out, idx_out, ws)
            self._pooled = (t0 + T) // self.m
        elif spec.kind == "window":
            q_pos = torch.arange(t0, t0 + T, dtype=torch.int64, device=q.device)
            ws = torch.empty(csa_workspace_size(p, OP_WINDOW_ATTN, 1, T, 0), dtype=torch.uint8,
                             device=q.device)
            window_attn(p, 1, T, q, self.x, self.n_raw, self.pos0, q_pos, sinks, out, ws)
        else:
            csa_compress(p, self.d, self.x[r0:r0 + n_pool], self.z[r0:r0 + n_pool], bias, n_pool,
                         _rows(self.kv, t0 // self.m, nb))
            self._pooled = (t0 + T) // self.m
            q_pos = torch.arange(t0, t0 + T, dtype=torch.int64, device=q.device)
            ws = torch.empty(csa_workspace_size(p, OP_HCA_ATTN, 1, T, self.cap_blocks),
                             dtype=torch.uint8, device=q.device)
            hca_attn(p, 1, T, q, self.kv, self.cap_blocks, self.x, self.n_raw, self.pos0, q_pos,
                     sinks, out, ws)


def _rows(st, j, n=1):
    """A view of rows [j, j + n) of a stored tensor (data and scales)."""
    from . import Stored
    return Stored(st.fmt, st.data[j:j + n], None if st.scales is None else st.scales[j:j + n])
