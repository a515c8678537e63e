"""Seeded synthetic inputs for the low-bit KV decode-attention step.

This module only draws random numbers; it holds none of the method's
arithmetic (no quantization, scoring, selection or merging), so both the
CUDA library's tests and the CPU oracle may take their inputs from it.

Workload shapes follow the decode-layer shapes named for the method
(Llama-3.1-8B, Qwen3-30B-A3B and Llama-70B attention layers, K3V2 and K4V4
caches; JetFire README, "benchmark" section).  The pages evaluate on
LongBench / NIAH with real model activations; those are not available, so
the recipe below stands in for them:

* q, K, V ~ N(0, 1), stored as bf16.
* Four key channels (drawn once per workload, shared by every head and token)
  are scaled by 10, imitating the outlier channels TailorKV's review
  describes (Section 3, Figure 2 there).
* ``planted`` tokens per sequence at distinct uniform positions in the
  quantized region; KV head ``h`` at planted slot ``j`` gets the key
  ``3 * q[h*G + (j mod G)] + N(0, 0.5)``, written after the outlier scaling.
  These stand in for needle tokens the approximate scan must find.
* Optionally (Qwen-shaped workload) every value row is multiplied by a
  per-token LogNormal(0, 0.5) factor.

Every segment (sequence ``b``, KV head ``h``) is drawn from its own
counter-derived seed, so any slice can be regenerated alone, on the CPU,
for sampled parity checks of large workloads.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator

import torch

HEAD_DIM = 128


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    kv_heads: int
    ctx: int
    key_bits: int
    val_bits: int
    topk: int
    planted: int
    seed: int = 0
    value_lognormal: bool = False
    head_dim: int = HEAD_DIM

    @property
    def group(self) -> int:
        return self.heads // self.kv_heads

    @property
    def n_quant(self) -> int:
        """Tokens in the quantized region (the tail keeps the last 1..64)."""
        return 0 if self.ctx <= 0 else 64 * ((self.ctx - 1) // 64)

    @property
    def fmt(self) -> str:
        return f"K{self.key_bits}V{self.val_bits}"

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sweep() -> list[Workload]:
    out = []
    for fmt in ((3, 2), (4, 4)):
        for ctx in (8192, 32768, 131072, 262144):
            for b in (1, 8, 32):
                out.append(Workload(
                    name=f"llama70b_k{fmt[0]}v{fmt[1]}_{ctx // 1024}k_b{b}",
                    batch=b, heads=64, kv_heads=8, ctx=ctx, key_bits=fmt[0],
                    val_bits=fmt[1], topk=256, planted=64,
                    seed=5_000 + 97 * ctx // 8192 + b + 7 * fmt[0]))
    return out


# Seeds: the tiny workload uses seed 0; the others use fixed per-workload
# offsets (recorded here) because the workload description leaves them open.
WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny_k4v4_4k", batch=1, heads=8, kv_heads=2, ctx=4096,
             key_bits=4, val_bits=4, topk=64, planted=16, seed=0),
    Workload("llama8b_k3v2_32k", batch=4, heads=32, kv_heads=8, ctx=32768,
             key_bits=3, val_bits=2, topk=256, planted=64, seed=1_000),
    Workload("llama8b_k4v4_128k", batch=1, heads=32, kv_heads=8, ctx=131072,
             key_bits=4, val_bits=4, topk=512, planted=64, seed=2_000),
    Workload("qwen30b_k3v2_32k", batch=16, heads=32, kv_heads=4, ctx=32768,
             key_bits=3, val_bits=2, topk=256, planted=64, seed=3_000,
             value_lognormal=True),
    *_sweep(),
]}

# The headline single-GPU workload (Llama-3.1-8B-shaped decode layer).
DEFAULT_WORKLOAD = "llama8b_k3v2_32k"


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _mix(*parts: int) -> int:
    """Counter-style seed derivation (splitmix64 finaliser over the parts)."""
    x = 0x9E37_79B9_7F4A_7C15
    for p in parts:
        x = (x ^ (int(p) & 0xFFFF_FFFF_FFFF_FFFF)) & 0xFFFF_FFFF_FFFF_FFFF
        x = (x + 0x9E37_79B9_7F4A_7C15) & 0xFFFF_FFFF_FFFF_FFFF
        x = ((x ^ (x >> 30)) * 0xBF58_476D_1CE4_E5B9) & 0xFFFF_FFFF_FFFF_FFFF
        x = ((x ^ (x >> 27)) * 0x94D0_49BB_1331_11EB) & 0xFFFF_FFFF_FFFF_FFFF
        x ^= x >> 31
    return x


def outlier_channels(w: Workload) -> torch.Tensor:
    return torch.randperm(w.head_dim, generator=_gen(_mix(w.seed, 1)))[:4]


def gen_q(w: Workload) -> torch.Tensor:
    """Query token of every sequence: bf16 [B, H, d]."""
    g = _gen(_mix(w.seed, 2))
    return torch.randn(w.batch, w.heads, w.head_dim, generator=g).to(torch.bfloat16)


def planted_positions(w: Workload, b: int) -> torch.Tensor:
    """Distinct planted-token positions of sequence b (shared by its KV heads)."""
    nq = w.n_quant
    n = min(w.planted, nq)
    if n == 0:
        return torch.zeros(0, dtype=torch.long)
    pos = torch.randperm(nq, generator=_gen(_mix(w.seed, 3, b)))[:n]
    return torch.sort(pos).values


def gen_segment(w: Workload, b: int, h: int, q: torch.Tensor | None = None,
                ctx: int | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Keys and values of sequence b, KV head h: two bf16 [ctx, d] tensors."""
    n = w.ctx if ctx is None else ctx
    d = w.head_dim
    if q is None:
        q = gen_q(w)
    g = _gen(_mix(w.seed, 4, b, h))
    k = torch.randn(n, d, generator=g)
    k[:, outlier_channels(w)] *= 10.0
    pos = planted_positions(w, b)
    pos = pos[pos < n]
    if pos.numel():
        j = torch.arange(pos.numel())
        src = q[b, h * w.group + (j % w.group)].float()
        k[pos] = 3.0 * src + 0.5 * torch.randn(pos.numel(), d, generator=g)
    v = torch.randn(n, d, generator=g)
    if w.value_lognormal:
        v *= torch.exp(0.5 * torch.randn(n, 1, generator=g))
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def gen_kv(w: Workload, q: torch.Tensor | None = None, ctx: int | None = None
           ) -> tuple[torch.Tensor, torch.Tensor]:
    """Whole cache as bf16 [B, H_kv, ctx, d] tensors (small workloads only)."""
    n = w.ctx if ctx is None else ctx
    if q is None:
        q = gen_q(w)
    k = torch.empty(w.batch, w.kv_heads, n, w.head_dim, dtype=torch.bfloat16)
    v = torch.empty_like(k)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            k[b, h], v[b, h] = gen_segment(w, b, h, q, n)
    return k, v


def segments(w: Workload) -> Iterator[tuple[int, int]]:
    for b in range(w.batch):
        for h in range(w.kv_heads):
            yield b, h


def sample_segments(w: Workload, n: int, seed: int = 0) -> list[tuple[int, int]]:
    """A deterministic sample of n (b, h) segments, always including (0, 0)
    and the last one."""
    total = w.batch * w.kv_heads
    if n >= total:
        return list(segments(w))
    g = _gen(_mix(w.seed, 5, seed))
    picks = set(torch.randperm(total, generator=g)[: max(0, n - 2)].tolist())
    picks |= {0, total - 1}
    return [(i // w.kv_heads, i % w.kv_heads) for i in sorted(picks)]


def default_scale(w: Workload) -> float:
    return 1.0 / math.sqrt(w.head_dim)


def gen_kv_device(w: Workload, device, q: torch.Tensor | None = None,
                  ctx: int | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """Same recipe as gen_kv, drawn with the device's generator (fast for large
    workloads).  Values differ from the CPU stream but are deterministic for
    a given seed; parity checks copy the sampled segments back to the host."""
    n = w.ctx if ctx is None else ctx
    d = w.head_dim
    if q is None:
        q = gen_q(w)
    qd = q.to(device)
    k = torch.empty(w.batch, w.kv_heads, n, d, dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k)
    outl = outlier_channels(w).to(device)
    g = torch.Generator(device=device)
    for b in range(w.batch):
        pos = planted_positions(w, b)
        pos = pos[pos < n].to(device)
        for h in range(w.kv_heads):
            g.manual_seed(_mix(w.seed, 6, b, h) & 0x7FFF_FFFF_FFFF_FFFF)
            kk = torch.randn(n, d, generator=g, device=device)
            kk[:, outl] *= 10.0
            if pos.numel():
                j = torch.arange(pos.numel(), device=device)
                src = qd[b, h * w.group + (j % w.group)].float()
                kk[pos] = 3.0 * src + 0.5 * torch.randn(pos.numel(), d, generator=g,
                                                        device=device)
            vv = torch.randn(n, d, generator=g, device=device)
            if w.value_lognormal:
                vv *= torch.exp(0.5 * torch.randn(n, 1, generator=g, device=device))
            k[b, h] = kk.to(torch.bfloat16)
            v[b, h] = vv.to(torch.bfloat16)
    return k, v
