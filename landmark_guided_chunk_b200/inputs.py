"""Seeded synthetic inputs for Hierarchical Sparse Attention (HSA).

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA library and the CPU oracle are fed from
here, so they always see identical tensors.

Workloads (the shapes the HSA pages talk about, "Every Token Counts 16m
Context", Core Technique / Implementation, and the value-of-information router
page for the gap-routed variant):

* ``tiny_f32``      prefill, fp32, B1 T4096 H2 Hkv2 d64 S64 k4
* ``prefill_bf16``  prefill, bf16, B1 T65536 H32 Hkv8 d128 S64 k16
* ``decode_1m``     decode,  bf16, B8, 1,048,576 cached tokens, H32 Hkv8 d128 S64 k16,
                    8 planted chunks per sequence
* ``router_bf16``   prefill, bf16, B1 T131072 H32 Hkv8 d128 S128 k8 (doubled to 16), tau 0.02
* ``decode_16m``    decode,  bf16, B1, 16,777,216 cached tokens, H32 Hkv8 d128 S64 k16,
                    4 planted chunks

Distributions: Q, K, V ~ N(0, 1); W_L ~ N(0, 1/d) for prefill and the identity
for decode (so that keys planted along the query direction show up in the
landmark score).  Values are drawn in fp32 and rounded (RNE) to the storage
dtype.  Draw order: Q, K, V, W_L, then planted positions and planted keys.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

__all__ = ["Problem", "WORKLOADS", "workload", "make_inputs", "make_output_grad", "torch_dtype"]


@dataclass(frozen=True)
class Problem:
    """Shape of one HSA call.  Tq query tokens sit at absolute positions
    q_pos0 .. q_pos0+Tq-1 over Tkv cached keys (prefill: Tq == Tkv, q_pos0 = 0;
    decode: Tq == 1, q_pos0 = Tkv)."""
    B: int
    Tq: int
    Tkv: int
    H: int
    Hkv: int
    d: int
    S: int
    k: int
    q_pos0: int = 0
    tau: float = 0.0
    dtype: str = "bf16"          # "f32" or "bf16"
    planted: int = 0             # decode workloads: planted chunks per sequence
    name: str = field(default="custom", compare=False)

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def C(self) -> int:
        """Complete chunks of the key sequence (a trailing partial chunk has no landmark)."""
        return self.Tkv // self.S

    @property
    def kmax(self) -> int:
        """Slots per (query, kv head) row in the selection outputs."""
        return 2 * self.k if self.tau > 0 else self.k

    @property
    def is_decode(self) -> bool:
        return self.Tq != self.Tkv or self.q_pos0 != 0

    def with_(self, **kw) -> "Problem":
        return replace(self, **kw)


def _prefill(name, B, T, H, Hkv, d, S, k, dtype, tau=0.0):
    return Problem(B=B, Tq=T, Tkv=T, H=H, Hkv=Hkv, d=d, S=S, k=k, q_pos0=0, tau=tau,
                   dtype=dtype, name=name)


def _decode(name, B, Tkv, H, Hkv, d, S, k, planted):
    return Problem(B=B, Tq=1, Tkv=Tkv, H=H, Hkv=Hkv, d=d, S=S, k=k, q_pos0=Tkv,
                   dtype="bf16", planted=planted, name=name)


WORKLOADS = {
    "tiny_f32": _prefill("tiny_f32", 1, 4096, 2, 2, 64, 64, 4, "f32"),
    "prefill_bf16": _prefill("prefill_bf16", 1, 65536, 32, 8, 128, 64, 16, "bf16"),
    "decode_1m": _decode("decode_1m", 8, 1 << 20, 32, 8, 128, 64, 16, planted=8),
    "router_bf16": _prefill("router_bf16", 1, 131072, 32, 8, 128, 128, 8, "bf16", tau=0.02),
    "decode_16m": _decode("decode_16m", 1, 1 << 24, 32, 8, 128, 64, 16, planted=4),
    # prefill_bf16 at head dim 64 (the tensor-core attention's other width)
    "prefill_bf16_d64": _prefill("prefill_bf16_d64", 1, 65536, 32, 8, 64, 64, 16, "bf16"),
}


def workload(name: str) -> Problem:
    return WORKLOADS[name]


def torch_dtype(dt: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dt]


def _randn_into(out: torch.Tensor, gen: torch.Generator, scale: float = 1.0,
                slice_elems: int = 1 << 28) -> None:
    """Fill ``out`` (contiguous) with N(0, scale^2) drawn in fp32 slice by slice
    and rounded to out's dtype, so big tensors never need an fp32 copy."""
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, slice_elems):
        e = min(n, s + slice_elems)
        x = torch.randn(e - s, generator=gen, device=out.device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[s:e].copy_(x)
        del x


def make_inputs(p: Problem, seed: int = 0, device: str | torch.device = "cpu") -> dict:
    """Draw Q [B,Tq,H,d], K and V [B,Tkv,Hkv,d], W_L [d,d] (row = input dim) and,
    for decode workloads with planted chunks, the planted chunk positions
    ``planted`` [B, n] (int64).  All tensors are contiguous, in p.dtype."""
    dev = torch.device(device)
    dt = torch_dtype(p.dtype)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    Q = torch.empty(p.B, p.Tq, p.H, p.d, dtype=dt, device=dev)
    K = torch.empty(p.B, p.Tkv, p.Hkv, p.d, dtype=dt, device=dev)
    V = torch.empty(p.B, p.Tkv, p.Hkv, p.d, dtype=dt, device=dev)
    _randn_into(Q, gen)
    _randn_into(K, gen)
    _randn_into(V, gen)
    if p.is_decode:
        W = torch.eye(p.d, dtype=dt, device=dev)
    else:
        W = torch.empty(p.d, p.d, dtype=dt, device=dev)
        _randn_into(W, gen, scale=1.0 / math.sqrt(p.d))
    out = {"Q": Q, "K": K, "V": V, "W_L": W}
    if p.planted > 0:
        out["planted"] = plant_chunks(p, Q, K, gen)
    return out


def make_output_grad(p: Problem, seed: int = 0, device: str | torch.device = "cpu") -> torch.Tensor:
    """An upstream gradient dO [B,Tq,H,d] ~ N(0, 1) in p.dtype for the backward
    (its own generator, so the forward inputs of the same seed are unchanged)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    dO = torch.empty(p.B, p.Tq, p.H, p.d, dtype=torch_dtype(p.dtype), device=dev)
    _randn_into(dO, gen)
    return dO


def plant_chunks(p: Problem, Q: torch.Tensor, K: torch.Tensor, gen: torch.Generator) -> torch.Tensor:
    """Overwrite the keys of ``p.planted`` distinct, uniformly placed chunks per
    sequence so that they point along the group query direction with cosine 0.9:
    for kv head j, u = qbar_j/|qbar_j| with qbar_j the sum of the group's query
    heads; every key of the chunk becomes |g| (0.9 u + sqrt(0.19) n) with
    g ~ N(0, I) and n a random unit vector orthogonal to u.  The positions are
    shared by all kv heads of a sequence."""
    dev = K.device
    C = p.C
    pos = torch.empty(p.B, p.planted, dtype=torch.int64, device=dev)
    for b in range(p.B):
        perm = torch.randperm(C, generator=gen, device=dev)
        pos[b] = perm[: p.planted].sort().values
    qbar = Q[:, -1].float().view(p.B, p.Hkv, p.G, p.d).sum(2)          # [B,Hkv,d]
    u = qbar / qbar.norm(dim=-1, keepdim=True)
    for b in range(p.B):
        for c in pos[b].tolist():
            g = torch.randn(p.S, p.Hkv, p.d, generator=gen, device=dev, dtype=torch.float32)
            n = torch.randn(p.S, p.Hkv, p.d, generator=gen, device=dev, dtype=torch.float32)
            ub = u[b].unsqueeze(0)                                      # [1,Hkv,d]
            n = n - (n * ub).sum(-1, keepdim=True) * ub
            n = n / n.norm(dim=-1, keepdim=True)
            key = g.norm(dim=-1, keepdim=True) * (0.9 * ub + math.sqrt(0.19) * n)
            K[b, c * p.S:(c + 1) * p.S].copy_(key.to(K.dtype))
    return pos
