"""The synthetic workloads: shapes, storage formats and value distributions.

Nothing here computes any step of the attention method; it only names the
tensors each workload needs, their shapes, and the N(0, std^2) stream each is
drawn from (see synth/__init__.py for the generator).  Quantised tensors are
described by their pre-quantisation values; each side quantises them with its
own quantiser.

Workloads (seed 0 unless a test says otherwise):
  csa_prefill_1k_fp32   one CSA layer prefill, fp32, T=1024, H=8, d=64, HI=4,
                        dI=32, m=4 (256 entries), k=16, W=64, scale 1/8
  csa_prefill_8k_bf16   CSA prefill, bf16, T=8192, H=64, d=512, HI=64, dI=128,
                        m=4 (2048 entries), k=512, W=128, scale 1/sqrt(512)
  csa_decode_128k_b32   CSA decode, B=32, 131072 context tokens, 1 query each;
                        32768 FP8 entries (E4M3 + scale per 64), MXFP4 indexer
                        keys and queries, 64 x 128; k=512, W=128 bf16 raw tokens
  hca_decode_1m_b8      HCA decode, B=8, 1,048,576 context tokens pooled at
                        m'=128 into 8192 FP8 entries; W=128, 64 heads x 512
Distributions: every tensor N(0,1) except the pooling bias B and the indexer
head weights w, which are N(0, 0.1^2).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

from . import tensor_np, tensor_torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_prefill" | "csa_decode" | "hca_decode"
    batch: int
    n_ctx: int           # decode: cached context tokens N (query at t = N); prefill: T
    H: int
    d: int
    HI: int
    dI: int
    m: int
    W: int
    k: int
    scale: float
    act: str             # "f32" | "bf16"
    kv: str              # "f32" | "bf16" | "fp8"
    idx: str             # "f32" | "bf16" | "mxfp4"
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def n_blocks(self) -> int:
        return self.n_ctx // self.m

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "csa_prefill_1k_fp32": Workload("csa_prefill_1k_fp32", "csa_prefill", 1, 1024, 8, 64, 4, 32,
                                    4, 64, 16, 1 / 8, "f32", "f32", "f32"),
    "csa_prefill_8k_bf16": Workload("csa_prefill_8k_bf16", "csa_prefill", 1, 8192, 64, 512, 64,
                                    128, 4, 128, 512, 1 / math.sqrt(512), "bf16", "bf16", "bf16"),
    "csa_decode_128k_b32": Workload("csa_decode_128k_b32", "csa_decode", 32, 131072, 64, 512, 64,
                                    128, 4, 128, 512, 1 / math.sqrt(512), "bf16", "fp8", "mxfp4"),
    "hca_decode_1m_b8": Workload("hca_decode_1m_b8", "hca_decode", 8, 1 << 20, 64, 512, 64, 128,
                                 128, 128, 0, 1 / math.sqrt(512), "bf16", "fp8", "mxfp4"),
}


def shapes(w: Workload) -> dict:
    """name -> (shape, std, storage dtype of the drawn values)."""
    B, H, d, HI, dI = w.batch, w.H, w.d, w.HI, w.dI
    a = "f32" if w.act == "f32" else "bf16"
    if w.kind == "csa_prefill":
        T = w.n_ctx
        return {
            "x": ((B, T, d), 1.0, a), "z": ((B, T, d), 1.0, a), "bias": ((w.m, d), 0.1, "f32"),
            "q": ((B, T, H, d), 1.0, a),
            "qI": ((B, T, HI, dI), 1.0, "f32" if w.idx in ("f32", "mxfp4") else "bf16"),
            "kI": ((B, T // w.m, dI), 1.0, "f32" if w.idx in ("f32", "mxfp4") else "bf16"),
            "w": ((B, T, HI), 0.1, "f32"), "sinks": ((H,), 1.0, "f32"),
        }
    if w.kind == "csa_decode":
        N = w.n_ctx
        return {
            "q": ((B, H, d), 1.0, a), "qI": ((B, HI, dI), 1.0, "f32"), "w": ((B, HI), 0.1, "f32"),
            "kv": ((B, N // w.m, d), 1.0, "f32"), "kI": ((B, N // w.m, dI), 1.0, "f32"),
            "window": ((B, w.W, d), 1.0, a), "sinks": ((H,), 1.0, "f32"),
        }
    if w.kind == "hca_decode":
        N = w.n_ctx
        return {
            "x": ((B, N, d), 1.0, a), "z": ((B, N, d), 1.0, a), "bias": ((w.m, d), 0.1, "f32"),
            "x_new": ((B, d), 1.0, a), "q": ((B, H, d), 1.0, a), "sinks": ((H,), 1.0, "f32"),
        }
    raise ValueError(w.kind)


def _stream_name(w: Workload, name: str) -> str:
    return f"{w.kind}/{name}"


def draw_np(w: Workload, name: str, batch_index: int | None = None):
    """Draw a tensor on the host (numpy).  With batch_index, only that
    sequence's slice (leading dimension) is drawn."""
    shape, std, dt = shapes(w)[name]
    if batch_index is None:
        return tensor_np(w.seed, _stream_name(w, name), shape, std, dt)
    per = 1
    for s in shape[1:]:
        per *= s
    return tensor_np(w.seed, _stream_name(w, name), shape[1:], std, dt, start=batch_index * per)


def draw_torch(w: Workload, name: str, device="cuda"):
    """Draw a tensor with torch on `device` (same stream as draw_np)."""
    shape, std, dt = shapes(w)[name]
    return tensor_torch(w.seed, _stream_name(w, name), shape, std, dt, device=device)
