"""CPU oracle for ClusterKV-style semantic cluster recall -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. It wraps ``libckv_oracle.so`` (plain C,
``ckv_oracle.c``) with numpy marshalling and a thread pool over independent
problems; the arithmetic lives entirely in the C file. It shares no code with
the CUDA path and never imports it.

Method source: "ClusterKV: Manipulating LLM KV Cache in Semantic Space for
Recallable Compression" (arXiv 2412.03213v2), section summaries on its
paperlayer.ai page: "III.B Clustering in the Semantic Space" (cosine k-means,
sinks, generated-token clustering), "IV.C Selection and Indexing" (metadata,
ranking, budget fill and trim), "III.A Problem Formulation and Design
Rationale" (top-B objective), "II.A LLM Inference and KV Cache" (attention).
"""
from __future__ import annotations

import ctypes
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

from . import build as _build

ROUND = {"none": 0, "f32": 1, "bf16": 2}
# clustering similarity ("III.B": cosine, with L2 and inner product as the
# paper's ablation)
METRIC = {"cos": 0, "ip": 1, "l2": 2}

_lib = None


def lib():
    global _lib
    if _lib is None:
        # CKV_ORACLE_LIB points the pins at another build of the oracle (the
        # mutation tests use it to show that planted mistakes are caught)
        path = os.environ.get("CKV_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C")
        c_int, c_sz, c_dbl = ctypes.c_int, ctypes.c_size_t, ctypes.c_double
        L.ckvo_bf16_bits.restype = ctypes.c_uint16
        L.ckvo_bf16_bits.argtypes = [c_dbl]
        L.ckvo_bf16_value.restype = c_dbl
        L.ckvo_bf16_value.argtypes = [ctypes.c_uint16]
        L.ckvo_init.argtypes = [f32p, c_int, c_int, c_int, c_int, f64p, f64p]
        L.ckvo_assign.argtypes = [f32p, c_int, c_int, f64p, c_int, i32p, ctypes.c_void_p]
        L.ckvo_update.argtypes = [f32p, c_int, c_int, i32p, c_int, c_int, f64p, f64p, i32p]
        L.ckvo_index.argtypes = [i32p, c_int, c_int, c_int, c_int, i32p, i32p]
        L.ckvo_kmeans.argtypes = [f32p, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                  f64p, f64p, i32p, i32p, i32p, i32p,
                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.ckvo_round.argtypes = [f64p, c_sz, c_int, f64p]
        L.ckvo_init_m.argtypes = [f32p, c_int, c_int, c_int, c_int, c_int, f64p, f64p]
        L.ckvo_assign_m.argtypes = [f32p, c_int, c_int, f64p, c_int, c_int, i32p,
                                    ctypes.c_void_p]
        L.ckvo_update_m.argtypes = [f32p, c_int, c_int, i32p, c_int, c_int, c_int, f64p, f64p,
                                    i32p]
        L.ckvo_kmeans_m.argtypes = [f32p, c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                    f64p, f64p, i32p, i32p, i32p, i32p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.ckvo_score.argtypes = [f32p, c_int, c_int, f32p, c_int, f32p]
        L.ckvo_select.restype = c_int
        L.ckvo_select.argtypes = [f32p, c_int, i32p, i32p, c_int, c_int, i32p]
        L.ckvo_selected_clusters.restype = c_int
        L.ckvo_selected_clusters.argtypes = [f32p, c_int, i32p, c_int, i32p, i32p]
        L.ckvo_cache_step.restype = c_int
        L.ckvo_cache_step.argtypes = [i32p, i32p, c_int, c_int, c_int, i32p, i32p,
                                      ctypes.POINTER(ctypes.c_int32)]
        L.ckvo_attend.argtypes = [f32p, c_int, c_int, f32p, f32p, i32p, c_int, c_dbl, f64p]
        L.ckvo_attended_rows.restype = c_int
        L.ckvo_attended_rows.argtypes = [c_int, i32p, c_int, c_int, c_int, i32p]
        _lib = L
    return _lib


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---- number formats ---------------------------------------------------------

def bf16_bits(x) -> np.ndarray:
    """Round-to-nearest-even bf16 bit patterns (uint16) of float64 values."""
    L = lib()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.fromiter((L.ckvo_bf16_bits(float(v)) for v in flat), dtype=np.uint16,
                      count=flat.size)
    return out.reshape(np.shape(x))


def bf16_value(bits) -> np.ndarray:
    """Values of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def round_to(x, mode: str) -> np.ndarray:
    x = _f64(x)
    out = np.empty_like(x)
    lib().ckvo_round(x.ravel(), x.size, ROUND[mode], out.ravel())
    return out


# ---- clustering --------------------------------------------------------------

def init(keys, C: int, mode: str, metric: str = "cos"):
    """Strided seeds mu and their assignment copy (mu/||mu|| for cosine, mu
    for "ip" and "l2"), rounded to `mode`."""
    keys = _f32(keys)
    n, d = keys.shape
    mu = np.zeros((C, d), np.float64)
    muhat = np.zeros((C, d), np.float64)
    if metric == "cos":
        lib().ckvo_init(keys, n, d, C, ROUND[mode], mu, muhat)
    else:
        lib().ckvo_init_m(keys, n, d, C, ROUND[mode], METRIC[metric], mu, muhat)
    return mu, muhat


def assign(keys, muhat, with_gap: bool = True, metric: str = "cos"):
    keys = _f32(keys)
    muhat = _f64(muhat)
    n, d = keys.shape
    labels = np.zeros(n, np.int32)
    gap = np.zeros(n, np.float64) if with_gap else None
    if metric == "cos":
        lib().ckvo_assign(keys, n, d, muhat, muhat.shape[0], labels, _ptr(gap))
    else:
        lib().ckvo_assign_m(keys, n, d, muhat, muhat.shape[0], METRIC[metric], labels,
                            _ptr(gap))
    return labels, gap


def update(keys, labels, mu, muhat, mode: str, metric: str = "cos"):
    keys = _f32(keys)
    mu = _f64(mu).copy()
    muhat = _f64(muhat).copy()
    n, d = keys.shape
    C = mu.shape[0]
    sizes = np.zeros(C, np.int32)
    if metric == "cos":
        lib().ckvo_update(keys, n, d, _i32(labels), C, ROUND[mode], mu, muhat, sizes)
    else:
        lib().ckvo_update_m(keys, n, d, _i32(labels), C, ROUND[mode], METRIC[metric], mu,
                            muhat, sizes)
    return mu, muhat, sizes


def index(labels, C: int, tok_begin: int, perm_base: int = 0):
    labels = _i32(labels)
    n = labels.size
    offsets = np.zeros(C + 1, np.int32)
    perm = np.zeros(n, np.int32)
    lib().ckvo_index(labels, n, C, tok_begin, perm_base, offsets, perm)
    return offsets, perm


def kmeans(keys, C: int, T: int, mode: str, tok_begin: int = 0, perm_base: int = 0,
           history: bool = False, metric: str = "cos") -> dict:
    """Strided init, T rounds of (assign, update), then the index (T >= 1)."""
    keys = _f32(keys)
    n, d = keys.shape
    if T < 1 or C < 1 or n < C:
        raise ValueError("need T >= 1 and 1 <= C <= n")
    r = dict(mu=np.zeros((C, d), np.float64), muhat=np.zeros((C, d), np.float64),
             labels=np.zeros(n, np.int32), sizes=np.zeros(C, np.int32),
             offsets=np.zeros(C + 1, np.int32), perm=np.zeros(n, np.int32))
    lh = mh = gh = None
    if history:
        lh = r["labels_hist"] = np.zeros((T, n), np.int32)
        mh = r["muhat_hist"] = np.zeros((T + 1, C, d), np.float64)
        gh = r["gap_hist"] = np.zeros((T, n), np.float64)
    if metric == "cos":
        lib().ckvo_kmeans(keys, n, d, C, T, ROUND[mode], tok_begin, perm_base, r["mu"],
                          r["muhat"], r["labels"], r["sizes"], r["offsets"], r["perm"], _ptr(lh),
                          _ptr(mh), _ptr(gh))
    else:
        lib().ckvo_kmeans_m(keys, n, d, C, T, ROUND[mode], METRIC[metric], tok_begin, perm_base,
                            r["mu"], r["muhat"], r["labels"], r["sizes"], r["offsets"],
                            r["perm"], _ptr(lh), _ptr(mh), _ptr(gh))
    return r


# ---- selection ---------------------------------------------------------------

def score(q, mu_lp) -> np.ndarray:
    """Cluster scores [C] (fp32) of the query heads q [G, d] against mu_lp [C, d]."""
    q = _f32(q)
    mu_lp = _f32(mu_lp)
    G, d = q.shape
    s = np.zeros(mu_lp.shape[0], np.float32)
    lib().ckvo_score(q, G, d, mu_lp, mu_lp.shape[0], s)
    return s


def select(s, offsets, perm, budget: int, perm_base: int = 0):
    s = _f32(s)
    offsets = _i32(offsets)
    perm = _i32(perm)
    sel = np.zeros(max(budget, 1), np.int32)
    cnt = lib().ckvo_select(s, s.size, offsets, perm, perm_base, budget, sel)
    return sel[:cnt].copy(), cnt


# ---- the cache of selected clusters ("D. Caching KV of Selected Tokens") -------

NEVER = -(1 << 30)  # last-selected step of a cluster that was never selected


def selected_clusters(s, offsets, budget: int):
    """The clusters a selection recalls, in rank order, and how many tokens of
    each are recalled."""
    s = _f32(s)
    offsets = _i32(offsets)
    C = s.size
    clusters = np.zeros(max(C, 1), np.int32)
    taken = np.zeros(max(C, 1), np.int32)
    m = lib().ckvo_selected_clusters(s, C, offsets, budget, clusters, taken)
    return clusters[:m].copy(), taken[:m].copy()


def cache_step(clusters, taken, step: int, R: int, last: np.ndarray):
    """One step of the cache of the last R steps' clusters; `last` (int32 [C],
    NEVER for never-selected clusters) is updated in place. Returns (hits,
    hit_tokens, misses in rank order)."""
    clusters = _i32(clusters)
    taken = _i32(taken)
    assert last.dtype == np.int32 and last.flags["C_CONTIGUOUS"]
    misses = np.zeros(max(clusters.size, 1), np.int32)
    ht = ctypes.c_int32(0)
    hits = lib().ckvo_cache_step(clusters, taken, clusters.size, step, R, last, misses,
                                 ctypes.byref(ht))
    return hits, int(ht.value), misses[:clusters.size - hits].copy()


# ---- attention ---------------------------------------------------------------

def attended_rows(sink: int, sel_idx, tail_begin: int, tail_end: int) -> np.ndarray:
    sel = _i32(sel_idx)
    rows = np.zeros(sink + sel.size + max(0, tail_end - tail_begin) + 1, np.int32)
    n = lib().ckvo_attended_rows(sink, sel, sel.size, tail_begin, tail_end, rows)
    return rows[:n].copy()


def attend(q, K, V, rows, scale: float) -> np.ndarray:
    """Attention of q [G, d] over rows of K, V [L, d]; double output [G, d]."""
    q = _f32(q)
    K = _f32(K)
    V = _f32(V)
    rows = _i32(rows)
    G, d = q.shape
    out = np.zeros((G, d), np.float64)
    lib().ckvo_attend(q, G, d, K, V, rows, rows.size, float(scale), out)
    return out


# ---- many independent problems ------------------------------------------------

def threads_default() -> int:
    return os.cpu_count() or 1


def map_problems(fn, items, threads: Optional[int] = None):
    """Run fn over independent problems on a thread pool (the C calls release
    the GIL), returning results in order."""
    threads = threads or threads_default()
    if threads <= 1 or len(items) <= 1:
        return [fn(x) for x in items]
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


__all__ = ["ROUND", "METRIC", "lib", "bf16_bits", "bf16_value", "round_to", "init", "assign", "update",
           "index", "kmeans", "score", "select", "selected_clusters", "cache_step", "NEVER",
           "attended_rows", "attend", "map_problems",
           "threads_default"]
