"""Seeded synthetic inputs shaped like the ClusterKV workloads.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It holds input generation only: nothing here clusters,
selects or attends.

Workload shapes follow the ClusterKV paper summary (arXiv 2412.03213v2):
32k-token prompts, head dimension 128, budgets of 1k-2k tokens
("V.C Inference Efficiency", "I. Introduction"), C0 = 400 prompt clusters
("V.B Model Accuracy") and 16 attention-sink tokens ("III.B Clustering in the
Semantic Space"). The paper's datasets (LongBench, PG19) are not available, so
keys come from a seeded mixture of random directions instead:

* per problem, M unit directions u_m = normalise(N(0, I_d));
* token i picks m_i uniformly in [0, M), draws per-channel noise
  e_i ~ N(0, sigma^2 I_d) and a norm s_i ~ U[0.5, 2], and its key is
  k_i = s_i * (u_m + e_i) / ||u_m + e_i||;
* each query head draws one query the same way from its KV head's mixture
  (optionally scaled, for a peaked softmax);
* values are N(0, 1);
* everything is rounded to the config's storage dtype (bf16 by
  round-to-nearest-even, or kept in fp32).

Generation runs on whatever torch device is asked for, one problem at a time,
so the 69 GB multi-layer workload can be produced directly in HBM. Each
problem has its own generator streams; a host copy of any problem has exactly
the same bits as the device tensor it came from.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, clustering and selection parameters."""

    name: str
    P: int              # independent (layer, batch, KV-head) problems
    G: int              # query heads per KV head
    L: int              # prompt length (tokens per problem after prefill)
    d: int              # head dimension
    dtype: str          # "bf16" or "f32"
    S: int              # attention-sink tokens
    W: int              # recent window kept dense after prefill
    C: int              # prompt clusters
    T: int              # k-means iterations
    B: int              # token budget
    M: int              # mixture components per problem
    sigma: float = 0.3  # per-channel noise of the mixture
    q_scale: float = 1.0
    steps: int = 1      # decode steps
    tail_cap: int = 0   # tail capacity that triggers incremental clustering (0: off)
    inc_C: int = 4      # clusters added per incremental clustering
    inc_T: int = 10     # iterations of incremental clustering
    layers: int = 1
    batch: int = 1
    heads_kv: int = 1
    seed: int = 0
    planted: bool = False  # clustered tokens drawn in M contiguous blocks (test variant)

    @property
    def N(self) -> int:
        """Tokens clustered at prefill: positions [S, L - W)."""
        return self.L - self.S - self.W

    @property
    def L_cap(self) -> int:
        """Rows reserved per problem in the K/V cache (prompt + appended tokens)."""
        return self.L + (self.steps if self.tail_cap else 0)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


SEED_BASE = 0xC1A5

# The five workloads, and one profiling stand-in. Problem index
# p = ((layer * batch + b) * heads_kv + h).
WORKLOADS = {
    # Tiny single head, fp32, 32-component mixture.
    "tiny_f32": Workload("tiny_f32", P=1, G=1, L=2048, d=128, dtype="f32", S=4, W=32,
                         C=32, T=10, B=256, M=32, seed=SEED_BASE + 1),
    # Llama-2-7B-shaped layer: batch 1, 32 KV heads, 32k context.
    "llama2_layer_32k": Workload("llama2_layer_32k", P=32, G=1, L=32768, d=128, dtype="bf16",
                                 S=16, W=64, C=400, T=10, B=1024, M=400,
                                 batch=1, heads_kv=32, seed=SEED_BASE + 2),
    # Llama-3-8B-shaped GQA layer: batch 8, 8 KV heads x 4 query heads.
    "llama3_gqa_32k": Workload("llama3_gqa_32k", P=64, G=4, L=32768, d=128, dtype="bf16",
                               S=16, W=64, C=400, T=10, B=2048, M=400,
                               batch=8, heads_kv=8, seed=SEED_BASE + 3),
    # Full 32-layer decode loop, Llama-2-7B shapes, batch 4; 256 decode steps,
    # incremental clustering of the filled recent window into 4 more clusters.
    "llama2_32layer_decode": Workload("llama2_32layer_decode", P=32 * 4 * 32, G=1, L=32768,
                                      d=128, dtype="bf16", S=16, W=64, C=400, T=10, B=1024,
                                      M=400, steps=256, tail_cap=320, inc_C=4, inc_T=10,
                                      layers=32, batch=4, heads_kv=32, seed=SEED_BASE + 4),
    # Long context: batch 4, 8 KV heads (4 query heads each), 128k tokens.
    "long_128k": Workload("long_128k", P=32, G=4, L=131072, d=128, dtype="bf16",
                          S=16, W=128, C=1600, T=8, B=2048, M=1600, steps=64,
                          batch=4, heads_kv=8, seed=SEED_BASE + 5),
    # Profiling stand-in for the many-problem decode (a problem per CTA):
    # 8 layers x batch 4 x 32 KV heads at 8k context, clusters of the same
    # average size (C = 100), so a capture holds ~4.5 GB instead of 69 GB.
    "llama2_8layer_8k_decode": Workload("llama2_8layer_8k_decode", P=8 * 4 * 32, G=1, L=8192,
                                        d=128, dtype="bf16", S=16, W=64, C=100, T=10, B=1024,
                                        M=100, layers=8, batch=4, heads_kv=32,
                                        seed=SEED_BASE + 6),
}

WORKLOAD_ORDER = ["tiny_f32", "llama2_layer_32k", "llama3_gqa_32k",
                  "llama2_32layer_decode", "long_128k"]


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    # one independent stream per (workload seed, tensor, problem)
    g.manual_seed((seed * 1_000_003 + stream * 7919) % (2**63 - 1))
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    n = torch.linalg.vector_norm(x, dim=-1, keepdim=True)
    return x / torch.clamp(n, min=1e-30)


def mixture_rows(dirs: torch.Tensor, n: int, sigma: float, g: torch.Generator,
                 scale: float = 1.0, comp: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Draw n rows per problem from the mixture with directions dirs [p, M, d] (fp32).

    comp [p, n] optionally fixes each row's component instead of drawing it."""
    p, M, d = dirs.shape
    drawn = torch.randint(0, M, (p, n), generator=g, device=dirs.device)
    comp = drawn if comp is None else comp
    noise = torch.randn((p, n, d), generator=g, device=dirs.device) * sigma
    x = torch.gather(dirs, 1, comp[..., None].expand(p, n, d)) + noise
    norms = torch.rand((p, n, 1), generator=g, device=dirs.device) * 1.5 + 0.5
    return _unit_rows(x) * norms * scale


def directions(w: Workload, p: int, device) -> torch.Tensor:
    """The M unit mixture directions [M, d] (fp32) of problem p."""
    g = _gen(device, w.seed, 1_000_000 + p)
    return _unit_rows(torch.randn((w.M, w.d), generator=g, device=device))


def make_kv(w: Workload, device="cpu", rows: Optional[int] = None,
            problems: Optional[Sequence[int]] = None,
            out_k: Optional[torch.Tensor] = None, out_v: Optional[torch.Tensor] = None):
    """Keys and values [len(problems), rows, d] in the workload's dtype.

    rows defaults to L_cap and problems to range(P). Every problem has its own
    generator streams, so any subset of problems can be regenerated alone on
    the same device with identical bits.
    """
    rows = w.L_cap if rows is None else rows
    problems = range(w.P) if problems is None else problems
    n = len(problems)
    dt = w.torch_dtype
    K = out_k if out_k is not None else torch.empty((n, rows, w.d), dtype=dt, device=device)
    V = out_v if out_v is not None else torch.empty((n, rows, w.d), dtype=dt, device=device)
    comp = None
    if w.planted:
        # the clustered rows [S, L - W) come in M equal contiguous blocks, so the
        # strided seeds land one per block when M divides N (a test variant)
        comp = torch.randint(0, w.M, (1, rows), device=device)
        j = torch.arange(w.S, w.L - w.W, device=device)
        comp[0, w.S:w.L - w.W] = (j - w.S) * w.M // w.N
    for i, p in enumerate(problems):
        dirs = directions(w, p, device)[None]
        gk = _gen(device, w.seed, 2_000_000 + p)
        K[i] = mixture_rows(dirs, rows, w.sigma, gk, comp=comp)[0].to(dt)
        gv = _gen(device, w.seed, 3_000_000 + p)
        V[i] = torch.randn((rows, w.d), generator=gv, device=device).to(dt)
    return K, V


def make_queries(w: Workload, step: int = 0, device="cpu",
                 problems: Optional[Sequence[int]] = None) -> torch.Tensor:
    """Decode queries [len(problems), G, d] for decode step `step`, each from its
    problem's mixture (scaled by q_scale)."""
    problems = range(w.P) if problems is None else problems
    out = torch.empty((len(problems), w.G, w.d), dtype=w.torch_dtype, device=device)
    for i, p in enumerate(problems):
        dirs = directions(w, p, device)[None]
        g = _gen(device, w.seed, 4_000_000 + 1_000_003 * step + p)
        out[i] = mixture_rows(dirs, w.G, w.sigma, g, scale=w.q_scale)[0].to(w.torch_dtype)
    return out


def directions_all(w: Workload, device) -> torch.Tensor:
    """Mixture directions of every problem, [P, M, d] (fp32)."""
    return torch.stack([directions(w, p, device) for p in range(w.P)])


def make_queries_batched(w: Workload, dirs: torch.Tensor, step: int) -> torch.Tensor:
    """Decode queries [P, G, d] for step `step` drawn for all problems at once
    from one generator stream per step (for long decode loops over many
    problems; a different stream than make_queries)."""
    g = _gen(dirs.device, w.seed, 6_000_000 + step)
    return mixture_rows(dirs, w.G, w.sigma, g, scale=w.q_scale).to(w.torch_dtype)


def correlated_queries(w: Workload, dirs: torch.Tensor, steps: int, rho: float) -> torch.Tensor:
    """A sequence of decode queries [steps, P, G, d] whose direction drifts:
    q_t = |q_{t-1}| * normalise(rho * u_{t-1} + sqrt(1 - rho^2) * e_t), with
    u_{t-1} = q_{t-1} / |q_{t-1}| and e_t the unit direction of a fresh mixture
    query (make_queries_batched), q_0 a fresh query. rho = 0 gives independent
    steps; rho -> 1 repeats the first query. Consecutive decode queries of a
    language model are correlated; the pages give no model of it, so this is a
    stand-in whose rho is a free parameter."""
    out = torch.empty((steps,) + tuple(dirs.shape[:1]) + (w.G, w.d), dtype=w.torch_dtype,
                      device=dirs.device)
    q = make_queries_batched(w, dirs, 0).float()
    out[0] = q.to(w.torch_dtype)
    a, b = float(rho), float((1.0 - rho * rho) ** 0.5)
    for t in range(1, steps):
        e = _unit_rows(make_queries_batched(w, dirs, t).float())
        nrm = torch.linalg.vector_norm(q, dim=-1, keepdim=True)
        q = nrm * _unit_rows(a * _unit_rows(q) + b * e)
        out[t] = q.to(w.torch_dtype)
    return out


def random_labels(P: int, n: int, C: int, seed: int, device="cpu",
                  skew: float = 0.0) -> torch.Tensor:
    """Seeded cluster labels [P, n] int32 in [0, C), for stage-level tests.

    skew > 0 draws from a Zipf-like law (some clusters large, some empty).
    """
    g = _gen(device, seed, 5_000_000)
    if skew <= 0:
        return torch.randint(0, C, (P, n), generator=g, device=device, dtype=torch.int32)
    w = torch.arange(1, C + 1, device=device, dtype=torch.float64) ** (-skew)
    idx = torch.multinomial(w.expand(P, C).contiguous(), n, replacement=True, generator=g)
    return idx.to(torch.int32)


def bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """Raw bf16 bit patterns of a bf16 tensor as uint16 (via int16 view)."""
    assert x.dtype == torch.bfloat16
    return x.contiguous().view(torch.int16)


def describe(w: Workload) -> dict:
    return {"workload": w.name, "P": w.P, "G": w.G, "L": w.L, "d": w.d, "dtype": w.dtype,
            "S": w.S, "W": w.W, "N": w.N, "C": w.C, "T": w.T, "B": w.B, "M": w.M,
            "sigma": w.sigma, "q_scale": w.q_scale, "steps": w.steps, "seed": w.seed}


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


__all__ = ["Workload", "WORKLOADS", "WORKLOAD_ORDER", "make_kv", "make_queries",
           "make_queries_batched", "directions_all", "random_labels", "mixture_rows",
           "directions", "describe", "ceil_div"]
