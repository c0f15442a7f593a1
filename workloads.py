"""Seeded synthetic decode workloads for SOCKET (inputs only).

This module draws the random inputs that both the CUDA library and the CPU
oracle consume: hyperplanes W, queries q and the key/value cache.  It holds
none of the method's arithmetic (no hashing, no soft assignment, no scoring,
no selection, no attention); the only vector algebra here builds the planted
"needle" keys at a chosen cosine to a query.

Shapes follow long-context decode of a Llama-3-8B-like layer (32 query heads,
8 kv heads, head dim 128) at the context lengths the SOCKET pages discuss
(32K to 128K, up to millions of tokens).  Every tensor is drawn from a
``torch.Generator`` seeded per workload, in a fixed order, on the device the
caller names.  CPU and CUDA generators give different streams, so a parity
test draws once, on one device, and hands the same tensors to both sides.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    L: int
    P: int
    tau: float
    k: int
    d: int = 128
    dtype: str = "bf16"                       # storage type of q, K, V ("bf16" | "f32")
    outlier_channels: tuple = ()              # channels of K and V scaled by outlier_scale
    outlier_scale: float = 8.0
    value_lognormal_sigma: float = 0.0        # v <- v * exp(sigma * g), g ~ N(0, 1) per row
    needles_per_head: int = 0                 # planted keys per query head
    needle_cosine: float = 0.9
    drift_per_block: float = 0.0              # k, v += drift * floor(pos / drift_block)
    drift_block: int = 131072
    appends: int = 0                          # decode steps that each append one key
    tau_sweep: tuple = ()
    seed: int = 0
    notes: str = field(default="", compare=False)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def U(self) -> int:
        """Independent (batch, kv-head) units."""
        return self.B * self.Hkv

    @property
    def ncap(self) -> int:
        """Cache capacity per unit: live keys plus appends, rounded up to 32."""
        return round_up(self.N + self.appends, 32)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def step_bytes(self, n: int | None = None) -> int:
        """Algorithmic HBM bytes of one decode step: per kv head, the bucket
        ids (L bytes per key), the fp32 value norms (4 bytes per key) and the
        k gathered key and value rows."""
        n = self.N if n is None else n
        return self.U * (n * self.L + 4 * n + 2 * self.k * self.d * self.elem_bytes)

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads.  Seeds are 1000 + workload number.
TINY = Workload(
    name="tiny_single_head_4k", B=1, Hq=1, Hkv=1, N=4096, L=16, P=4, tau=0.5, k=256,
    dtype="f32", seed=1001,
    notes="single head, fp32 q/K/V ~ N(0,1)")
LLAMA_32K = Workload(
    name="llama8b_layer_32k", B=1, Hq=32, Hkv=8, N=32768, L=60, P=8, tau=0.3, k=2048,
    outlier_channels=(0, 1, 2, 3), value_lognormal_sigma=0.5, seed=1002,
    notes="bf16 K/V ~ N(0,1), channels 0-3 x8, value norms lognormal(0.5)")
BATCH8_128K = Workload(
    name="batch8_128k", B=8, Hq=32, Hkv=8, N=131072, L=32, P=8, tau=0.3, k=2048,
    outlier_channels=(0, 1, 2, 3), value_lognormal_sigma=0.5, needles_per_head=16, seed=1003,
    notes="as llama8b_layer_32k plus 16 needles per query head at cosine 0.9")
MILLION = Workload(
    name="million_token_1m", B=1, Hq=32, Hkv=8, N=1048576, L=32, P=8, tau=0.2, k=4096,
    drift_per_block=0.5, seed=1004,
    notes="bf16 K/V ~ N(0,1), mean +0.5 every 131072 positions")
APPEND_MIX = Workload(
    name="batch32_16k_append64", B=32, Hq=32, Hkv=8, N=16384, L=60, P=8, tau=0.5, k=1024,
    appends=64, tau_sweep=(1.0, 0.1, 0.01), seed=1005,
    notes="prefill hash of 16384 keys, then 64 steps each appending one key")

WORKLOADS = {w.name: w for w in (TINY, LLAMA_32K, BATCH8_128K, MILLION, APPEND_MIX)}
ORDER = [TINY, LLAMA_32K, BATCH8_128K, MILLION, APPEND_MIX]


def _unit_vector_orthogonal(r: torch.Tensor, qhat: torch.Tensor) -> torch.Tensor:
    u = r - (r * qhat).sum(-1, keepdim=True) * qhat
    return u / u.norm(dim=-1, keepdim=True)


@torch.no_grad()
def make_inputs(w: Workload, device="cpu", batches=None):
    """Draw every input of workload ``w`` on ``device``.

    Returns a dict with
      W      [L, P, d] bf16          hyperplanes, N(0, 1) rounded to bf16
      q      [B, Hq, d]              decode queries (storage dtype)
      K, V   [B, Hkv, ncap, d]       key / value cache (storage dtype)
      q_steps [appends, B, Hq, d]    one query per append step (if appends)
      needles [B, Hkv, G*needles]    planted positions per kv head (if needles)
    ``batches`` (an iterable of batch rows) restricts K and V to those rows;
    the random stream is still consumed for every row so values do not change.
    """
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    dt = w.torch_dtype
    d, ncap = w.d, w.ncap

    W = torch.randn(w.L, w.P, d, generator=g, device=device).to(torch.bfloat16)
    q = torch.randn(w.B, w.Hq, d, generator=g, device=device).to(dt)

    keep = list(range(w.B)) if batches is None else sorted(set(int(b) for b in batches))
    K = torch.empty(len(keep), w.Hkv, ncap, d, dtype=dt, device=device)
    V = torch.empty_like(K)
    needles = torch.empty(len(keep), w.Hkv, w.G * w.needles_per_head, dtype=torch.int64, device=device)
    pos = torch.arange(ncap, device=device, dtype=torch.float32)
    last = max(keep)
    for b in range(w.B):
        if b > last and not w.appends:
            break  # later rows only consume the stream; nothing drawn after them is needed
        Kb = torch.randn(w.Hkv, ncap, d, generator=g, device=device)
        Vb = torch.randn(w.Hkv, ncap, d, generator=g, device=device)
        if w.outlier_channels:
            ch = list(w.outlier_channels)
            Kb[..., ch] *= w.outlier_scale
            Vb[..., ch] *= w.outlier_scale
        factor = None
        if w.value_lognormal_sigma:
            factor = torch.exp(w.value_lognormal_sigma * torch.randn(w.Hkv, ncap, generator=g, device=device))
        if w.drift_per_block:
            shift = w.drift_per_block * torch.floor(pos / w.drift_block)
            Kb += shift[None, :, None]
            Vb += shift[None, :, None]
        if w.needles_per_head:
            m = w.needles_per_head
            qb = q[b].float()                                  # [Hq, d]
            qhat = qb / qb.norm(dim=-1, keepdim=True)
            for kvh in range(w.Hkv):
                where = torch.randperm(w.N, generator=g, device=device)[: w.G * m]
                r = torch.randn(w.G * m, d, generator=g, device=device)
                heads = kvh * w.G + torch.arange(w.G * m, device=device) // m
                qh = qhat[heads]                               # [G*m, d]
                u = _unit_vector_orthogonal(r, qh)
                c = w.needle_cosine
                norms = Kb[kvh, where].norm(dim=-1, keepdim=True)
                Kb[kvh, where] = norms * (c * qh + math.sqrt(1.0 - c * c) * u)
                if factor is not None:
                    factor[kvh, where] = 1.0
                if b in keep:
                    needles[keep.index(b), kvh] = where
        if factor is not None:
            Vb *= factor[..., None]
        if b in keep:
            K[keep.index(b)] = Kb.to(dt)
            V[keep.index(b)] = Vb.to(dt)
        del Kb, Vb
    out = {"W": W, "q": q, "K": K, "V": V, "batches": keep}
    if w.needles_per_head:
        out["needles"] = needles
    if w.appends:
        out["q_steps"] = torch.randn(w.appends, w.B, w.Hq, d, generator=g, device=device).to(dt)
    return out
