"""Shared helpers of the test suite: seeded inputs, oracle calls per problem,
and comparison rules. Imports the oracle (test infrastructure) and the
binding; nothing here is used by the product path."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from semantic_cluster_recall_b200 import synth

# Tolerances (the path's stated bars):
GAP_EXEMPT = 1e-4      # labels may differ only where the oracle's top-2 cosine gap is below this
CENT_REL_L2 = 1e-3     # per-centroid relative L2 error of mu
OUT_MAX_ABS = 2e-3     # attention output, max-abs error (bf16 in, fp32 accumulate)


def mode_of(dtype: torch.dtype) -> str:
    return "bf16" if dtype == torch.bfloat16 else "f32"


def f32np(t: torch.Tensor) -> np.ndarray:
    """Exact float32 host copy (bf16 -> fp32 is exact)."""
    return t.detach().float().cpu().numpy()


def to_dev(x: np.ndarray, dtype: torch.dtype, device) -> torch.Tensor:
    """Values already representable in dtype, to the device in dtype."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dtype)
    assert np.array_equal(t.float().numpy(), np.asarray(x, dtype=np.float32)), "not representable"
    return t.to(device)


def small_workload(dtype=torch.bfloat16, P=3, G=1, L=3000, S=16, W=64, C=50, T=4, B=300, M=None,
                   sigma=0.3, q_scale=1.0, seed=1234) -> synth.Workload:
    return synth.Workload(name="small", P=P, G=G, L=L, d=128,
                          dtype="bf16" if dtype == torch.bfloat16 else "f32", S=S, W=W, C=C,
                          T=T, B=B, M=M or C, sigma=sigma, q_scale=q_scale, seed=seed)


def oracle_kmeans_all(Kh: np.ndarray, w: synth.Workload, history=False, threads=None):
    """Oracle clustering of positions [S, L - W) of every problem of Kh [P, rows, d]."""
    mode = w.dtype
    tb, te = w.S, w.L - w.W

    def run(p):
        return oracle.kmeans(Kh[p, tb:te], w.C, w.T, mode, tok_begin=tb, history=history)

    return oracle.map_problems(run, list(range(Kh.shape[0])), threads)


def labels_match_except_near_ties(gpu: np.ndarray, ref: np.ndarray, gap: np.ndarray,
                                  tol=GAP_EXEMPT):
    diff = gpu != ref
    bad = diff & (gap >= tol)
    return int(diff.sum()), int(bad.sum()), int((gap < tol).sum())


def centroid_rel_err(gpu: np.ndarray, ref: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(gpu.astype(np.float64) - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return num / np.maximum(den, 1e-30)


def scale_of(d: int) -> float:
    return 1.0 / math.sqrt(d)
