"""Device-memory holder and call sequencing for the three C-ABI stages.

ClusterRecall owns the caller-side buffers that libckv needs (centroids,
cluster index, selections, workspaces) as torch CUDA tensors and sequences the
entry points of ckv.py for a batch of P independent (layer, batch, KV-head)
problems:

* prefill(K): cosine k-means of positions [S, L - W) of every problem
  ("III.B Clustering in the Semantic Space" of "ClusterKV: Manipulating LLM KV
  Cache in Semantic Space for Recallable Compression", arXiv 2412.03213v2);
* select(q): cluster-granularity recall under the token budget ("IV.C
  Selection and Indexing");
* decode(q): attention over sinks + recalled + recent tokens;
* append(k, v) / incremental(): one generated token per step, and clustering
  of the oldest generated tokens into a few new clusters once the recent tail
  reaches its capacity ("III.B": generated tokens are clustered on their own
  into four new centroids every so many steps);
* incremental_begin() / incremental_commit(): the same clustering started
  early on a side stream, behind the decode steps of the main stream, and
  published later ("IV.B Semantic Clustering": clustering is launched
  asynchronously and overlaps other inference work). Until the commit the
  steps read only the committed clusters; the new ones are written to
  metadata slots no step reads.

Nothing here computes: every step is one of libckv's kernels.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import ckv


class ClusterRecall:
    def __init__(self, P: int, G: int, d: int, dtype: torch.dtype, kv_rows: int, S: int,
                 budget: int, C_cap: int, perm_cap: int, max_tail: int, device,
                 stream: Optional[torch.cuda.Stream] = None):
        if d != 128:
            raise ValueError("d must be 128")
        self.P, self.G, self.d, self.dtype = P, G, d, dtype
        self.kv_rows, self.S, self.B = kv_rows, S, budget
        self.C_cap, self.perm_cap, self.max_tail = C_cap, perm_cap, max_tail
        self.device = torch.device(device)
        self.stream = stream
        dev = self.device
        i32 = torch.int32
        self.centroids = torch.zeros((P, C_cap, d), dtype=torch.float32, device=dev)
        self.centroids_hat = torch.zeros((P, C_cap, d), dtype=dtype, device=dev)
        self.centroids_lp = torch.zeros((P, C_cap, d), dtype=dtype, device=dev)
        self.sizes = torch.zeros((P, C_cap), dtype=i32, device=dev)
        self.offsets = torch.zeros((P, C_cap + 1), dtype=i32, device=dev)
        self.labels = torch.zeros((P, perm_cap), dtype=i32, device=dev)
        self.perm = torch.zeros((P, perm_cap), dtype=i32, device=dev)
        self.n_clusters = torch.zeros((P,), dtype=i32, device=dev)
        self.tail_begin = torch.zeros((P,), dtype=i32, device=dev)
        self.tail_end = torch.zeros((P,), dtype=i32, device=dev)
        self.sel_idx = torch.zeros((P, max(budget, 1)), dtype=i32, device=dev)
        self.sel_cnt = torch.zeros((P,), dtype=i32, device=dev)
        self.out = torch.zeros((P, G, d), dtype=torch.float32, device=dev)
        self.ws_select = ckv.workspace(ckv.ckv_select_workspace_bytes(P, C_cap), dev)
        self.ws_decode = ckv.workspace(
            ckv.ckv_decode_workspace_bytes(P, G, d, S + budget + max_tail), dev)
        self.ws_cluster: Optional[torch.Tensor] = None
        # host-side bookkeeping of the clustered region (same for all problems)
        self.n_clustered = 0      # perm slots used
        self.C_used = 0           # clusters used
        self.tail_lo = 0          # host copy of tail_begin (uniform over problems)
        self.scale = 1.0 / math.sqrt(d)
        self._pending = None      # background clustering in flight: (n_tok, C, end, event)
        self.cache_R: Optional[int] = None  # cache of the last R steps' clusters, if enabled

    def _main(self):
        return self.stream if self.stream is not None else torch.cuda.current_stream(self.device)

    def _ws_cluster(self, n_tok: int, C: int) -> torch.Tensor:
        need = ckv.ckv_cluster_workspace_bytes(self.P, n_tok, C)
        if self.ws_cluster is None or self.ws_cluster.numel() < need:
            self.ws_cluster = ckv.workspace(need, self.device)
        return self.ws_cluster

    def prefill(self, K: torch.Tensor, L: int, W: int, C: int, iters: int):
        """Cluster positions [S, L - W); the last W prompt tokens start the tail."""
        tb, te = self.S, L - W
        ws = self._ws_cluster(te - tb, C)
        ckv.ckv_cluster(K, K.stride(0), tb, te, C, iters, 0, 0, self.C_cap, self.perm_cap,
                        self.centroids, self.centroids_hat, self.centroids_lp, self.labels,
                        self.sizes, self.offsets, self.perm, ws, P=self.P, d=self.d,
                        stream=self.stream)
        self.n_clustered, self.C_used, self.tail_lo = te - tb, C, te
        with torch.cuda.stream(self._main()):
            self.n_clusters.fill_(C)
            self.tail_begin.fill_(te)
            self.tail_end.fill_(L)

    def prefill_from_host(self, K_host: torch.Tensor, V_host: torch.Tensor, K: torch.Tensor,
                          V: torch.Tensor, L: int, W: int, C: int, iters: int,
                          copy_stream: torch.cuda.Stream, groups: int = 8):
        """prefill() for K and V that start in pinned host memory: the problems
        are uploaded in `groups` groups on copy_stream, and each group is
        clustered on the main stream as soon as its keys have arrived, so the
        host-to-device copy (the bound here) overlaps the clustering. Values
        follow the keys (only decoding reads them); the main stream waits for
        them before returning. Rows [0, L) of every problem are copied."""
        P = self.P
        groups = max(1, min(groups, P))
        main = self._main()
        tb, te = self.S, L - W
        ws = self._ws_cluster(te - tb, C)
        start = torch.cuda.Event()
        start.record(main)
        copy_stream.wait_event(start)  # after everything queued before this call
        bounds = [P * g // groups for g in range(groups + 1)]
        arrived = []
        with torch.cuda.stream(copy_stream):
            for g in range(groups):
                a, b = bounds[g], bounds[g + 1]
                K[a:b, :L].copy_(K_host[a:b, :L], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_stream)
                arrived.append(ev)
            V[:, :L].copy_(V_host[:, :L], non_blocking=True)
            v_done = torch.cuda.Event()
            v_done.record(copy_stream)
        for g in range(groups):
            a, b = bounds[g], bounds[g + 1]
            if a == b:
                continue
            main.wait_event(arrived[g])
            ckv.ckv_cluster(K[a:b], K.stride(0), tb, te, C, iters, 0, 0, self.C_cap,
                            self.perm_cap, self.centroids[a:b], self.centroids_hat[a:b],
                            self.centroids_lp[a:b], self.labels[a:b], self.sizes[a:b],
                            self.offsets[a:b], self.perm[a:b], ws, P=b - a, d=self.d,
                            stream=main)
        main.wait_event(v_done)
        self.n_clustered, self.C_used, self.tail_lo = te - tb, C, te
        with torch.cuda.stream(main):
            self.n_clusters.fill_(C)
            self.tail_begin.fill_(te)
            self.tail_end.fill_(L)

    def incremental(self, K: torch.Tensor, n_tok: int, C: int, iters: int):
        """Cluster the oldest n_tok tail tokens into C new clusters appended to
        the metadata; the tail then starts after them."""
        tb, te = self.tail_lo, self.tail_lo + n_tok
        ws = self._ws_cluster(n_tok, C)
        ckv.ckv_cluster(K, K.stride(0), tb, te, C, iters, self.C_used, self.n_clustered,
                        self.C_cap, self.perm_cap, self.centroids, self.centroids_hat,
                        self.centroids_lp, self.labels, self.sizes, self.offsets, self.perm, ws,
                        P=self.P, d=self.d, stream=self.stream)
        self.n_clustered += n_tok
        self.C_used += C
        self.tail_lo = te
        with torch.cuda.stream(self._main()):
            self.n_clusters.fill_(self.C_used)
            self.tail_begin.fill_(te)

    def incremental_begin(self, K: torch.Tensor, n_tok: int, C: int, iters: int,
                          side_stream: torch.cuda.Stream, max_sms: int = 0):
        """Start clustering the oldest n_tok tail tokens into C new clusters on
        side_stream, after the work queued so far on the main stream (the
        appends that wrote those tokens). The persistent assignment kernel is
        held to max_sms SMs (0 = all), so that a low-priority side stream
        leaves the rest of the GPU to the decode steps."""
        if self._pending is not None:
            raise RuntimeError("a background clustering is already in flight")
        tb, te = self.tail_lo, self.tail_lo + n_tok
        ws = self._ws_cluster(n_tok, C)
        ws.record_stream(side_stream)
        ready = torch.cuda.Event()
        ready.record(self._main())
        side_stream.wait_event(ready)
        ckv.ckv_cluster_ex(K, K.stride(0), tb, te, C, iters, self.C_used, self.n_clustered,
                           self.C_cap, self.perm_cap, self.centroids, self.centroids_hat,
                           self.centroids_lp, self.labels, self.sizes, self.offsets, self.perm,
                           ws, max_sms=max_sms, P=self.P, d=self.d, stream=side_stream)
        done = torch.cuda.Event()
        done.record(side_stream)
        self._pending = (n_tok, C, te, done)

    def incremental_commit(self):
        """Publish the clusters of incremental_begin(): the main stream waits
        for the side stream's work, then the steps see the new clusters and
        the tail starts after their tokens."""
        if self._pending is None:
            raise RuntimeError("no background clustering in flight")
        n_tok, C, te, done = self._pending
        main = self._main()
        main.wait_event(done)
        self.n_clustered += n_tok
        self.C_used += C
        self.tail_lo = te
        with torch.cuda.stream(main):
            self.n_clusters.fill_(self.C_used)
            self.tail_begin.fill_(te)
        self._pending = None

    def select(self, q: torch.Tensor):
        ckv.ckv_select(q, self.centroids_lp, self.n_clusters, self.C_cap, self.offsets, self.perm,
                       self.perm_cap, self.B, self.sel_idx, self.sel_cnt, self.ws_select,
                       P=self.P, G=self.G, d=self.d, stream=self.stream)

    def decode(self, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor) -> torch.Tensor:
        ckv.ckv_sparse_decode(q, K, V, K.stride(0), self.kv_rows, self.S, self.tail_begin,
                              self.tail_end, self.max_tail, self.sel_idx, self.sel_cnt, self.B,
                              self.scale, self.out, self.ws_decode, P=self.P, G=self.G,
                              d=self.d, stream=self.stream)
        return self.out

    def enable_cache(self, R: int):
        """Account a cache of the clusters selected in the last R steps ("D.
        Caching KV of Selected Tokens"): every later step(..., step_no=t)
        records per problem the hits, the selected clusters, the recalled
        tokens of the hits and all recalled tokens in cache_stats, and the
        clusters to load in miss_list."""
        P, dev = self.P, self.device
        self.cache_R = int(R)
        self.last_sel = torch.full((P, self.C_cap), ckv.NEVER_SELECTED, dtype=torch.int32,
                                   device=dev)
        self.cache_stats = torch.zeros((P, 4), dtype=torch.int32, device=dev)
        self.miss_list = torch.zeros((P, self.C_cap), dtype=torch.int32, device=dev)

    def step(self, q, K, V, step_no: Optional[int] = None) -> torch.Tensor:
        """One decode step: selection then sparse attention, as one fused
        launch (ckv_select_decode) when the shape allows it; with the cache
        enabled, also its accounting for step number step_no."""
        if self.cache_R is not None:
            if step_no is None or self.G not in (1, 2, 4):
                raise ValueError("a cached step needs step_no and G in (1, 2, 4)")
            ckv.ckv_select_decode_cached(q, self.centroids_lp, self.n_clusters, self.C_cap,
                                         self.offsets, self.perm, self.perm_cap, self.B,
                                         self.sel_idx, self.sel_cnt, K, V, K.stride(0),
                                         self.kv_rows, self.S, self.tail_begin, self.tail_end,
                                         self.max_tail, self.scale, self.out, self.last_sel,
                                         step_no, self.cache_R, self.cache_stats, self.miss_list,
                                         P=self.P, G=self.G, d=self.d, stream=self.stream)
            return self.out
        if self.G in (1, 2, 4):
            ckv.ckv_select_decode(q, self.centroids_lp, self.n_clusters, self.C_cap,
                                  self.offsets, self.perm, self.perm_cap, self.B, self.sel_idx,
                                  self.sel_cnt, K, V, K.stride(0), self.kv_rows, self.S,
                                  self.tail_begin, self.tail_end, self.max_tail, self.scale,
                                  self.out, P=self.P, G=self.G, d=self.d, stream=self.stream)
            return self.out
        self.select(q)
        return self.decode(q, K, V)

    def append(self, K, V, new_k, new_v):
        ckv.ckv_append(K, V, K.stride(0), self.kv_rows, new_k, new_v, self.tail_end, P=self.P,
                       d=self.d, stream=self.stream)
