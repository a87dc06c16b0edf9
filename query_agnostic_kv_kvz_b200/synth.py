"""Seeded synthetic inputs for the KVzip hot path (shapes of the workloads the
KVzip page evaluates: Llama-3.1-8B- and Qwen2.5-14B-shaped GQA caches).

This module only draws random numbers and shapes them; it contains none of
the scoring, selection or compaction arithmetic, so both the CUDA path and
the CPU oracle can be fed from it.  The model weights and the long-context
datasets the pages use are not available, so Q/K/V are drawn from simple
distributions with the stated shapes:

* Q, K_ctx, K_in, V i.i.d. N(0, 1), drawn in fp32 and rounded to bf16 with
  round-to-nearest-even;
* optionally a per-head key-channel scale sigma_c = exp(N(0, 0.5^2)) applied to
  channel c of both K_ctx and K_in (anisotropic keys, as real key caches have
  a few large channels);
* optionally "sink" keys: the first ``sinks`` context keys get 8 * u added,
  u the unit vector of the head's mean query row;
* optionally exact duplicate keys: floor(dup_frac * n_c) positions in
  [sinks, n_c) copy the bf16 bits of another (non-duplicate) position.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

__all__ = ["Workload", "WORKLOADS", "layer_inputs", "chunked_inputs", "synthetic_scores", "seed_for"]


@dataclass(frozen=True)
class Workload:
    """One benchmark/parity workload: a GQA cache shape plus a keep rule."""

    name: str
    L: int
    H: int
    G: int
    d: int
    n_c: Tuple[int, ...]          # one entry per context (ragged batches: several)
    n_prompt: int
    ratio: float
    mode: str                     # "per_head" | "global" | "heads" (head-level eviction)
    key_scale: bool = False       # per-channel log-normal key scale
    row_chunk: int = 0            # input rows per scoring pass (0 = all)
    in_place: bool = False        # compact K/V in place
    sinks: int = 0
    dup_frac: float = 0.0
    chunk: int = 0                # context chunk length m of chunked scoring (0 = unchunked)
    n_protect: int = 0            # leading positions of every head always kept (system prompt)
    quant: bool = False           # compact into an int8 cache with per-row scales
    extra: dict = field(default_factory=dict)

    def n_in(self, ctx: int = 0) -> int:
        return self.n_prompt + self.n_c[ctx]

    @property
    def B(self) -> int:
        return self.L * self.H


WORKLOADS = {
    "tiny": Workload("tiny", L=1, H=1, G=4, d=64, n_c=(256,), n_prompt=16,
                     ratio=0.3, mode="per_head"),
    "llama8b_layer": Workload("llama8b_layer", L=1, H=8, G=4, d=128, n_c=(8192,),
                              n_prompt=32, ratio=0.3, mode="per_head", key_scale=True),
    "llama8b_stack": Workload("llama8b_stack", L=32, H=8, G=4, d=128, n_c=(32768,),
                              n_prompt=32, ratio=0.3, mode="global", key_scale=True),
    "qwen14b_128k": Workload("qwen14b_128k", L=48, H=8, G=5, d=128, n_c=(131072,),
                             n_prompt=32, ratio=0.25, mode="per_head", key_scale=True,
                             row_chunk=4096, in_place=True),
    # head-level eviction: the 256 heads of the stack scored on an 8K context,
    # the best half kept whole
    "llama8b_stack_heads": Workload("llama8b_stack_heads", L=32, H=8, G=4, d=128, n_c=(8192,),
                                    n_prompt=32, ratio=0.5, mode="heads", key_scale=True),
    # a 64-token system prompt kept intact, the rest compacted into int8
    "llama8b_stack_int8": Workload("llama8b_stack_int8", L=32, H=8, G=4, d=128, n_c=(32768,),
                                   n_prompt=32, ratio=0.3, mode="global", key_scale=True,
                                   n_protect=64, quant=True),
    # chunked scoring: 2K-token chunks of a 170K context (83 full chunks + 16)
    "llama8b_170k_chunked": Workload("llama8b_170k_chunked", L=1, H=8, G=4, d=128, n_c=(170000,),
                                     n_prompt=32, ratio=0.3, mode="per_head", key_scale=True, chunk=2048),
    "stress_ragged": Workload("stress_ragged", L=32, H=8, G=4, d=128,
                              n_c=(1000, 17000, 65537, 170000), n_prompt=32,
                              ratio=0.1, mode="global", key_scale=True,
                              sinks=4, dup_frac=0.01),
}


def seed_for(workload: Workload, layer: int, ctx: int = 0, seed: int = 0) -> int:
    """Deterministic 63-bit seed of one (workload, context, layer) draw."""
    h = 1469598103934665603
    for part in (workload.name.encode(), str(ctx).encode(), str(layer).encode(),
                 str(seed).encode()):
        for byte in part:
            h ^= byte
            h = (h * 1099511628211) & ((1 << 64) - 1)
        h ^= 0xFF
        h = (h * 1099511628211) & ((1 << 64) - 1)
    return h & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def layer_inputs(workload: Workload, layer: int = 0, ctx: int = 0, seed: int = 0,
                 device="cpu", heads: Optional[int] = None,
                 n_c: Optional[int] = None, n_prompt: Optional[int] = None,
                 G: Optional[int] = None, d: Optional[int] = None):
    """Q/K_ctx/K_in/V (bf16) of one layer: shapes [H,G,n_in,d], [H,n_c,d],
    [H,n_in,d], [H,n_c,d].  Keyword overrides shrink a workload's shape while
    keeping its value distributions (used for small parity cases)."""
    H = workload.H if heads is None else heads
    G = workload.G if G is None else G
    d = workload.d if d is None else d
    n_c = workload.n_c[ctx] if n_c is None else n_c
    n_prompt = workload.n_prompt if n_prompt is None else n_prompt
    n_in = n_prompt + n_c
    g = _gen(device, seed_for(workload, layer, ctx, seed))
    f32 = torch.float32
    Q = torch.randn((H, G, n_in, d), generator=g, device=device, dtype=f32)
    K_ctx = torch.randn((H, n_c, d), generator=g, device=device, dtype=f32)
    K_in = torch.randn((H, n_in, d), generator=g, device=device, dtype=f32)
    V = torch.randn((H, n_c, d), generator=g, device=device, dtype=f32)
    if workload.key_scale:
        sigma = torch.exp(0.5 * torch.randn((H, 1, d), generator=g, device=device, dtype=f32))
        K_ctx.mul_(sigma)
        K_in.mul_(sigma)
    Q = Q.to(torch.bfloat16)
    if workload.sinks:
        mean_q = Q.float().reshape(H, G * n_in, d).mean(dim=1)          # [H, d]
        u = mean_q / mean_q.norm(dim=1, keepdim=True).clamp_min(1e-30)
        s = min(workload.sinks, n_c)
        K_ctx[:, :s, :] += 8.0 * u[:, None, :]
    K_ctx = K_ctx.to(torch.bfloat16)
    if workload.dup_frac > 0.0:
        ndup = int(workload.dup_frac * n_c)
        lo = min(workload.sinks, n_c)
        if ndup > 0 and n_c - lo > ndup:
            for h in range(H):
                perm = torch.randperm(n_c - lo, generator=g, device=device) + lo
                dst = perm[:ndup]
                pool = torch.cat([torch.arange(lo, device=device), perm[ndup:]])
                pick = torch.randint(0, pool.numel(), (ndup,), generator=g, device=device)
                K_ctx[h, dst] = K_ctx[h, pool[pick]]
    return {
        "Q": Q.contiguous(),
        "K_ctx": K_ctx.contiguous(),
        "K_in": K_in.to(torch.bfloat16).contiguous(),
        "V": V.to(torch.bfloat16).contiguous(),
    }


def synthetic_scores(B: int, n_c: int, seed: int = 0, device="cpu",
                     tie_frac: float = 0.05, special: bool = True) -> torch.Tensor:
    """fp32 scores [B, n_c] in [0, 1] with exact ties, zeros, subnormals and a
    few +inf entries, for exercising selection in isolation."""
    g = _gen(device, (seed * 2654435761 + 12345) & ((1 << 63) - 1))
    S = torch.rand((B, n_c), generator=g, device=device, dtype=torch.float32) ** 3
    flat = S.view(-1)
    n = flat.numel()
    nt = int(tie_frac * n)
    if nt > 0:
        src = torch.randint(0, n, (nt,), generator=g, device=device)
        dst = torch.randint(0, n, (nt,), generator=g, device=device)
        flat[dst] = flat[src]
    if special and n >= 16:
        k = max(1, n // 1000)
        pos = torch.randint(0, n, (4 * k,), generator=g, device=device)
        flat[pos[:k]] = 0.0
        flat[pos[k:2 * k]] = float("inf")
        flat[pos[2 * k:3 * k]] = 1e-42          # subnormal
        flat[pos[3 * k:]] = -0.0                # equal to +0
    return S


def chunked_inputs(workload: Workload, layer: int = 0, ctx: int = 0, seed: int = 0, device="cpu",
                   heads: Optional[int] = None, n_c: Optional[int] = None, n_prompt: Optional[int] = None,
                   G: Optional[int] = None, d: Optional[int] = None, m: Optional[int] = None):
    """Inputs of chunked scoring for one layer (bf16): every context chunk of m
    tokens is appended to the repeat prompt and has its own queries and input
    keys.  Returns Q [H, T, G, n_prompt+m, d] and K_in [H, T, n_prompt+m, d]
    for the T = n_c // m full chunks, Q_tail [H, G, n_prompt+m_last, d] and
    K_in_tail [H, n_prompt+m_last, d] for the shorter last chunk (None when m
    divides n_c), K_ctx and V [H, n_c, d].  Same distributions as
    layer_inputs (N(0,1); the key-channel scale on every key)."""
    H = workload.H if heads is None else heads
    G = workload.G if G is None else G
    d = workload.d if d is None else d
    n_c = workload.n_c[ctx] if n_c is None else n_c
    n_prompt = workload.n_prompt if n_prompt is None else n_prompt
    m = workload.chunk if m is None else m
    T, m_last = n_c // m, n_c % m
    g = _gen(device, seed_for(workload, layer, ctx, seed))
    f32 = torch.float32
    Q = torch.randn((H, T, G, n_prompt + m, d), generator=g, device=device, dtype=f32)
    K_in = torch.randn((H, T, n_prompt + m, d), generator=g, device=device, dtype=f32)
    Q_tail = torch.randn((H, G, n_prompt + m_last, d), generator=g, device=device, dtype=f32) if m_last else None
    K_in_tail = torch.randn((H, n_prompt + m_last, d), generator=g, device=device, dtype=f32) if m_last else None
    K_ctx = torch.randn((H, n_c, d), generator=g, device=device, dtype=f32)
    V = torch.randn((H, n_c, d), generator=g, device=device, dtype=f32)
    if workload.key_scale:
        sigma = torch.exp(0.5 * torch.randn((H, 1, d), generator=g, device=device, dtype=f32))
        K_ctx.mul_(sigma)
        K_in.mul_(sigma[:, None])
        if K_in_tail is not None:
            K_in_tail.mul_(sigma)
    bf = lambda t: None if t is None else t.to(torch.bfloat16).contiguous()
    return {"Q": bf(Q), "Q_tail": bf(Q_tail), "K_ctx": bf(K_ctx), "K_in": bf(K_in), "K_in_tail": bf(K_in_tail),
            "V": bf(V), "m": m}
