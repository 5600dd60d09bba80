"""Thin ctypes binding of libckv.so (include/ckv.h).

Each function has the name of the C entry point it calls and only marshals
arguments: torch tensors become device pointers, the stream becomes the
current torch CUDA stream's handle, and a non-OK status raises CkvError.
Every step of the computation runs in libckv's CUDA kernels; there is no
fallback. If the library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libckv.so")

CKV_OK, CKV_ERR_INVALID, CKV_ERR_CUDA, CKV_ERR_TIMEOUT, CKV_ERR_UNSUPPORTED = range(5)
CKV_F32, CKV_BF16 = 0, 1
CKV_DEVERR_LABEL, CKV_DEVERR_PERM, CKV_DEVERR_INDEX, CKV_DEVERR_OFFSETS = 1, 2, 4, 8
CKV_DEVERR_TIMEOUT = 0x10
MAX_CLUSTERS = 4096

# every entry point declared in include/ckv.h
EXPORTS = [
    "ckv_status_string", "ckv_last_error", "ckv_version", "ckv_device_error",
    "ckv_index_workspace_bytes", "ckv_cluster_workspace_bytes", "ckv_cluster",
    "ckv_init_centroids", "ckv_assign", "ckv_index", "ckv_update",
    "ckv_select_workspace_bytes", "ckv_select",
    "ckv_decode_workspace_bytes", "ckv_sparse_decode", "ckv_append",
    "ckv_sparse_decode_noalloc_scratch_bytes", "ckv_sparse_decode_noalloc",
    "ckv_select_decode", "ckv_cluster_ex", "ckv_cluster_ex_workspace_bytes",
    "ckv_init_centroids_ex", "ckv_assign_ex", "ckv_update_ex", "ckv_select_decode_cached",
    "ckv_selftest_timeout",
]
NOALLOC_SCRATCH_BYTES = 8 << 20


class CkvError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({_status_name(status)}): {detail}")
        self.status = status


def _status_name(s: int) -> str:
    return {0: "ok", 1: "invalid argument", 2: "CUDA error", 3: "timeout",
            4: "unsupported"}.get(s, "unknown")


_lib = None


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libckv.so (built in-tree by semantic_cluster_recall_b200.build)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libckv.so not found at {p}: build it with "
                           "`python -m semantic_cluster_recall_b200.build`")
    L = ctypes.CDLL(p)
    vp, i32, i64, sz, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                             ctypes.c_float)
    sig = {
        "ckv_status_string": (ctypes.c_char_p, [i32]),
        "ckv_last_error": (ctypes.c_char_p, []),
        "ckv_version": (i32, []),
        "ckv_device_error": (i32, [ctypes.POINTER(ctypes.c_uint), i32, vp]),
        "ckv_index_workspace_bytes": (sz, [i32, i32, i32]),
        "ckv_cluster_workspace_bytes": (sz, [i32, i32, i32]),
        "ckv_cluster": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32, i32, i32, i32,
                              vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ckv_cluster_ex": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32, i32, i32, i32,
                                 vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, i32, vp]),
        "ckv_cluster_ex_workspace_bytes": (sz, [i32, i32, i32, i32]),
        "ckv_init_centroids_ex": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32,
                                        vp, vp, vp, i32, vp, vp]),
        "ckv_assign_ex": (i32, [vp, i32, i32, i64, i32, i32, i32, vp, i32, i32, i32, vp, i32,
                                i32, vp, vp]),
        "ckv_update_ex": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32, vp, vp, i32,
                                vp, vp, vp, vp, i32, vp, vp]),
        "ckv_init_centroids": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32,
                                     vp, vp, vp, vp]),
        "ckv_assign": (i32, [vp, i32, i32, i64, i32, i32, i32, vp, i32, i32, i32, vp, i32, i32,
                             vp]),
        "ckv_index": (i32, [vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp]),
        "ckv_update": (i32, [vp, i32, i32, i64, i32, i32, i32, i32, i32, i32, vp, vp, i32,
                             vp, vp, vp, vp, vp]),
        "ckv_select_workspace_bytes": (sz, [i32, i32]),
        "ckv_select": (i32, [vp, i32, i32, i32, i32, vp, vp, i32, vp, vp, i32, i32, vp, vp,
                             vp, sz, vp]),
        "ckv_decode_workspace_bytes": (sz, [i32, i32, i32, i32]),
        "ckv_sparse_decode": (i32, [vp, vp, vp, i32, i32, i32, i32, i64, i32, i32, vp, vp, i32,
                                    vp, vp, i32, f32, vp, vp, sz, vp]),
        "ckv_append": (i32, [vp, vp, i32, i32, i32, i64, i32, vp, vp, vp, vp]),
        "ckv_sparse_decode_noalloc_scratch_bytes": (sz, [i32, i32, i32, i32]),
        "ckv_select_decode": (i32, [vp, i32, i32, i32, i32, vp, vp, i32, vp, vp, i32, i32, vp, vp,
                                    vp, vp, i64, i32, i32, vp, vp, i32, f32, vp, vp]),
        "ckv_select_decode_cached": (i32, [vp, i32, i32, i32, i32, vp, vp, i32, vp, vp, i32, i32,
                                           vp, vp, vp, vp, i64, i32, i32, vp, vp, i32, f32, vp,
                                           vp, i32, i32, vp, vp, vp]),
        "ckv_selftest_timeout": (i32, [ctypes.c_uint, vp]),
        "ckv_sparse_decode_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, i64, i32, i32, vp,
                                            vp, i32, vp, vp, i32, f32, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = L
    return L


def _check(status: int, where: str):
    if status != CKV_OK:
        detail = load().ckv_last_error().decode()
        raise CkvError(status, where, detail)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        if not torch.cuda.is_available():
            return None
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return CKV_BF16
    if t.dtype == torch.float32:
        return CKV_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- workspace sizes ---------------------------------------------------------------

def ckv_cluster_workspace_bytes(P: int, n_tok: int, C: int) -> int:
    return int(load().ckv_cluster_workspace_bytes(P, n_tok, C))


def ckv_index_workspace_bytes(P: int, n_tok: int, C: int) -> int:
    return int(load().ckv_index_workspace_bytes(P, n_tok, C))


def ckv_select_workspace_bytes(P: int, C_cap: int) -> int:
    return int(load().ckv_select_workspace_bytes(P, C_cap))


def ckv_decode_workspace_bytes(P: int, G: int, d: int, max_rows: int) -> int:
    return int(load().ckv_decode_workspace_bytes(P, G, d, max_rows))


def workspace(nbytes: int, device) -> torch.Tensor:
    """A caller-owned workspace buffer (torch allocations are 256-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---- entry points ------------------------------------------------------------------

def ckv_cluster(keys, problem_stride, tok_begin, tok_end, C, iters, cluster_base, perm_base,
                C_cap, perm_cap, centroids, centroids_hat, centroids_lp, labels, sizes,
                offsets, perm, ws, P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_cluster(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin, tok_end,
                            C, iters, cluster_base, perm_base, C_cap, perm_cap, _p(centroids),
                            _p(centroids_hat), _p(centroids_lp), _p(labels), _p(sizes),
                            _p(offsets), _p(perm), _p(ws), ws.numel() * ws.element_size(),
                            _stream(stream))
    _check(st, "ckv_cluster")


METRICS = {"cos": 0, "ip": 1, "l2": 2}  # ckv_metric: CKV_COSINE, CKV_INNER, CKV_L2


def ckv_cluster_ex_workspace_bytes(P: int, n_tok: int, C: int, metric: str = "cos") -> int:
    return int(load().ckv_cluster_ex_workspace_bytes(P, n_tok, C, METRICS[metric]))


def ckv_cluster_ex(keys, problem_stride, tok_begin, tok_end, C, iters, cluster_base, perm_base,
                   C_cap, perm_cap, centroids, centroids_hat, centroids_lp, labels, sizes,
                   offsets, perm, ws, metric="cos", max_sms=0, P=None, d=128, stream=None):
    """ckv_cluster under a similarity ("cos", "ip", "l2"), with the persistent
    assignment kernel held to max_sms SMs (0 = all) for clustering in the
    background beside other GPU work."""
    P = keys.shape[0] if P is None else P
    st = load().ckv_cluster_ex(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin,
                               tok_end, C, iters, cluster_base, perm_base, C_cap, perm_cap,
                               _p(centroids), _p(centroids_hat), _p(centroids_lp), _p(labels),
                               _p(sizes), _p(offsets), _p(perm), _p(ws),
                               ws.numel() * ws.element_size(), METRICS[metric], int(max_sms),
                               _stream(stream))
    _check(st, "ckv_cluster_ex")


def ckv_init_centroids_ex(keys, problem_stride, tok_begin, tok_end, C, cluster_base, C_cap,
                          centroids, centroids_hat, centroids_lp, metric="cos", bias=None,
                          P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_init_centroids_ex(_p(keys), dtype_code(keys), P, problem_stride, d,
                                      tok_begin, tok_end, C, cluster_base, C_cap, _p(centroids),
                                      _p(centroids_hat), _p(centroids_lp), METRICS[metric],
                                      _p(bias), _stream(stream))
    _check(st, "ckv_init_centroids_ex")


def ckv_assign_ex(keys, problem_stride, tok_begin, tok_end, centroids_hat, C, cluster_base,
                  C_cap, labels, perm_base, perm_cap, bias=None, P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_assign_ex(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin,
                              tok_end, _p(centroids_hat), C, cluster_base, C_cap, _p(labels),
                              perm_base, perm_cap, _p(bias), _stream(stream))
    _check(st, "ckv_assign_ex")


def ckv_update_ex(keys, problem_stride, tok_begin, tok_end, C, cluster_base, C_cap, offsets,
                  perm, perm_cap, centroids, centroids_hat, centroids_lp, sizes, metric="cos",
                  bias=None, P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_update_ex(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin,
                              tok_end, C, cluster_base, C_cap, _p(offsets), _p(perm), perm_cap,
                              _p(centroids), _p(centroids_hat), _p(centroids_lp), _p(sizes),
                              METRICS[metric], _p(bias), _stream(stream))
    _check(st, "ckv_update_ex")


def ckv_init_centroids(keys, problem_stride, tok_begin, tok_end, C, cluster_base, C_cap,
                       centroids, centroids_hat, centroids_lp, P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_init_centroids(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin,
                                   tok_end, C, cluster_base, C_cap, _p(centroids),
                                   _p(centroids_hat), _p(centroids_lp), _stream(stream))
    _check(st, "ckv_init_centroids")


def ckv_assign(keys, problem_stride, tok_begin, tok_end, centroids_hat, C, cluster_base, C_cap,
               labels, perm_base, perm_cap, P=None, d=128, stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_assign(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin, tok_end,
                           _p(centroids_hat), C, cluster_base, C_cap, _p(labels), perm_base,
                           perm_cap, _stream(stream))
    _check(st, "ckv_assign")


def ckv_index(labels, P, tok_begin, tok_end, C, cluster_base, C_cap, perm_base, perm_cap,
              offsets, perm, ws, stream=None):
    st = load().ckv_index(_p(labels), P, tok_begin, tok_end, C, cluster_base, C_cap, perm_base,
                          perm_cap, _p(offsets), _p(perm), _p(ws),
                          ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "ckv_index")


def ckv_update(keys, problem_stride, tok_begin, tok_end, C, cluster_base, C_cap, offsets, perm,
               perm_cap, centroids, centroids_hat, centroids_lp, sizes, P=None, d=128,
               stream=None):
    P = keys.shape[0] if P is None else P
    st = load().ckv_update(_p(keys), dtype_code(keys), P, problem_stride, d, tok_begin, tok_end,
                           C, cluster_base, C_cap, _p(offsets), _p(perm), perm_cap,
                           _p(centroids), _p(centroids_hat), _p(centroids_lp), _p(sizes),
                           _stream(stream))
    _check(st, "ckv_update")


def ckv_select(q, centroids_lp, n_clusters, C_cap, offsets, perm, perm_cap, budget, sel_idx,
               sel_cnt, ws, P=None, G=None, d=128, stream=None):
    P = q.shape[0] if P is None else P
    G = q.shape[1] if G is None else G
    st = load().ckv_select(_p(q), dtype_code(q), P, G, d, _p(centroids_lp), _p(n_clusters),
                           C_cap, _p(offsets), _p(perm), perm_cap, budget, _p(sel_idx),
                           _p(sel_cnt), _p(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "ckv_select")


def ckv_select_decode(q, centroids_lp, n_clusters, C_cap, offsets, perm, perm_cap, budget,
                      sel_idx, sel_cnt, K, V, kv_problem_stride, kv_rows, sink, tail_begin,
                      tail_end, max_tail, scale, out, P=None, G=None, d=128, stream=None):
    P = q.shape[0] if P is None else P
    G = q.shape[1] if G is None else G
    st = load().ckv_select_decode(_p(q), dtype_code(q), P, G, d, _p(centroids_lp),
                                  _p(n_clusters), C_cap, _p(offsets), _p(perm), perm_cap, budget,
                                  _p(sel_idx), _p(sel_cnt), _p(K), _p(V), kv_problem_stride,
                                  kv_rows, sink, _p(tail_begin), _p(tail_end), max_tail,
                                  float(scale), _p(out), _stream(stream))
    _check(st, "ckv_select_decode")


def ckv_selftest_timeout(limit_us: int, stream=None):
    """Make one bounded device wait give up (a flag nothing sets); the next
    ckv_device_error reports the timeout."""
    _check(load().ckv_selftest_timeout(int(limit_us), _stream(stream)), "ckv_selftest_timeout")


NEVER_SELECTED = -(1 << 30)  # last-selected step of a cluster no step selected


def ckv_select_decode_cached(q, centroids_lp, n_clusters, C_cap, offsets, perm, perm_cap, budget,
                             sel_idx, sel_cnt, K, V, kv_problem_stride, kv_rows, sink, tail_begin,
                             tail_end, max_tail, scale, out, last_sel, step, R, cache_stats,
                             miss_list=None, P=None, G=None, d=128, stream=None):
    """ckv_select_decode plus the accounting of a cache of the clusters
    selected in the last R steps (last_sel: int32 [P][C_cap], initialised to
    NEVER_SELECTED; cache_stats: int32 [P][4])."""
    P = q.shape[0] if P is None else P
    G = q.shape[1] if G is None else G
    st = load().ckv_select_decode_cached(
        _p(q), dtype_code(q), P, G, d, _p(centroids_lp), _p(n_clusters), C_cap, _p(offsets),
        _p(perm), perm_cap, budget, _p(sel_idx), _p(sel_cnt), _p(K), _p(V), kv_problem_stride,
        kv_rows, sink, _p(tail_begin), _p(tail_end), max_tail, float(scale), _p(out),
        _p(last_sel), int(step), int(R), _p(cache_stats), _p(miss_list), _stream(stream))
    _check(st, "ckv_select_decode_cached")


def ckv_sparse_decode(q, K, V, kv_problem_stride, kv_rows, sink, tail_begin, tail_end, max_tail,
                      sel_idx, sel_cnt, budget, scale, out, ws, P=None, G=None, d=128,
                      stream=None):
    P = q.shape[0] if P is None else P
    G = q.shape[1] if G is None else G
    st = load().ckv_sparse_decode(_p(q), _p(K), _p(V), dtype_code(q), P, G, d, kv_problem_stride,
                                  kv_rows, sink, _p(tail_begin), _p(tail_end), max_tail,
                                  _p(sel_idx), _p(sel_cnt), budget, float(scale), _p(out), _p(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "ckv_sparse_decode")


def ckv_sparse_decode_noalloc(q, K, V, kv_problem_stride, kv_rows, sink, tail_begin, tail_end,
                              max_tail, sel_idx, sel_cnt, budget, scale, out, P=None, G=None,
                              d=128, stream=None):
    """ckv_sparse_decode without a workspace, for callers that cannot allocate
    device memory: the library's fixed scratch array holds the partials (see
    include/ckv.h for the size limit and for the rule that overlapping calls
    race on that array)."""
    P = q.shape[0] if P is None else P
    G = q.shape[1] if G is None else G
    st = load().ckv_sparse_decode_noalloc(_p(q), _p(K), _p(V), dtype_code(q), P, G, d,
                                          kv_problem_stride, kv_rows, sink, _p(tail_begin),
                                          _p(tail_end), max_tail, _p(sel_idx), _p(sel_cnt),
                                          budget, float(scale), _p(out), _stream(stream))
    _check(st, "ckv_sparse_decode_noalloc")


def ckv_sparse_decode_noalloc_scratch_bytes(P: int, G: int, d: int, max_rows: int) -> int:
    return int(load().ckv_sparse_decode_noalloc_scratch_bytes(P, G, d, max_rows))


def ckv_append(K, V, kv_problem_stride, kv_rows, new_k, new_v, tail_end, P=None, d=128,
               stream=None):
    P = new_k.shape[0] if P is None else P
    st = load().ckv_append(_p(K), _p(V), dtype_code(K), P, d, kv_problem_stride, kv_rows,
                           _p(new_k), _p(new_v), _p(tail_end), _stream(stream))
    _check(st, "ckv_append")


def ckv_device_error(clear: bool = True, stream=None) -> int:
    flags = ctypes.c_uint(0)
    st = load().ckv_device_error(ctypes.byref(flags), int(clear), _stream(stream))
    _check(st, "ckv_device_error")
    return int(flags.value)
