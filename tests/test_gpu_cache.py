"""The cache of the clusters selected in the last R decode steps.

"D. Caching KV of Selected Tokens" of "ClusterKV: Manipulating LLM KV Cache in
Semantic Space for Recallable Compression": the GPU cache retains the KV and
cluster labels selected in the last R decoding steps and loads only clusters
absent from it; the paper reports average cluster hit rates of 63% (R = 1)
and 74% (R = 2) on real decoding.

The fused step's accounting (ckv_select_decode_cached) must agree with the
oracle step by step: the same hits, selected clusters, recalled tokens of the
hits and the same clusters to load, in rank order, for every problem, with
the selection and the attention unchanged. The oracle's centroids and index
feed both sides; the queries drift from step to step.
"""
import numpy as np
import pytest
import torch

import oracle
from semantic_cluster_recall_b200 import ckv, synth
from semantic_cluster_recall_b200.pipeline import ClusterRecall

from helpers import OUT_MAX_ABS, f32np

pytestmark = pytest.mark.gpu


def _state(w, dev, K):
    """ClusterRecall holding the oracle's clustering of every problem."""
    tb, te = w.S, w.L - w.W
    n = te - tb
    st = ClusterRecall(w.P, w.G, w.d, w.torch_dtype, w.L_cap, w.S, w.B, w.C, n, w.W, dev)
    Kh = f32np(K)
    mode = w.dtype
    lp = np.zeros((w.P, w.C, w.d), np.float32)
    off = np.zeros((w.P, w.C + 1), np.int32)
    perm = np.zeros((w.P, n), np.int32)

    def run(p):
        return p, oracle.kmeans(Kh[p, tb:te], w.C, 3, mode, tok_begin=tb)

    for p, r in oracle.map_problems(run, list(range(w.P))):
        lp[p] = oracle.round_to(r["mu"], mode)
        off[p], perm[p] = r["offsets"], r["perm"]
    st.centroids_lp.copy_(torch.from_numpy(lp))
    st.offsets.copy_(torch.from_numpy(off))
    st.perm.copy_(torch.from_numpy(perm))
    st.n_clusters.fill_(w.C)
    st.tail_begin.fill_(te)
    st.tail_end.fill_(w.L)
    return st, lp, off, perm


@pytest.mark.parametrize("R,rho,G", [(1, 0.9, 1), (2, 0.9, 4), (0, 0.95, 2), (1, 0.0, 1)])
def test_cache_accounting_matches_oracle(cuda_device, R, rho, G):
    dev = cuda_device
    w = synth.WORKLOADS["llama2_layer_32k"].replace(P=6, G=G, L=6000, C=75, B=700, M=75,
                                                     seed=321 + R)
    K, V = synth.make_kv(w, device=dev)
    st, lp, off, perm = _state(w, dev, K)
    st.enable_cache(R)
    dirs = synth.directions_all(w, dev)
    qs = synth.correlated_queries(w, dirs, 10, rho)
    last = np.full((w.P, w.C), oracle.NEVER, np.int32)
    Kh, Vh = f32np(K), f32np(V)
    te = w.L - w.W
    total_hits = 0
    for step in range(qs.shape[0]):
        q = qs[step]
        out = st.step(q, K, V, step_no=step)
        torch.cuda.synchronize()
        stats = st.cache_stats.cpu().numpy()
        miss = st.miss_list.cpu().numpy()
        sel, cnt, o = st.sel_idx.cpu().numpy(), st.sel_cnt.cpu().numpy(), out.cpu().numpy()
        qh = f32np(q)
        for p in range(w.P):
            s = oracle.score(qh[p], lp[p])
            ref_sel, ref_cnt = oracle.select(s, off[p], perm[p], w.B)
            assert cnt[p] == ref_cnt and np.array_equal(sel[p, :ref_cnt], ref_sel)
            cl, taken = oracle.selected_clusters(s, off[p], w.B)
            hits, ht, misses = oracle.cache_step(cl, taken, step, R, last[p])
            assert tuple(stats[p]) == (hits, cl.size, ht, ref_cnt), (step, p)
            assert np.array_equal(miss[p, :cl.size - hits], misses), (step, p)
            total_hits += hits
            rows = oracle.attended_rows(w.S, ref_sel, te, w.L)
            att = oracle.attend(qh[p], Kh[p], Vh[p], rows, 1 / np.sqrt(w.d))
            assert np.abs(o[p] - att).max() <= OUT_MAX_ABS
        assert np.array_equal(st.last_sel.cpu().numpy()[:, :w.C], last)
    assert ckv.ckv_device_error() == 0
    if R == 0:
        assert total_hits == 0
    elif rho >= 0.9:
        assert total_hits > 0


def test_cache_off_is_the_plain_step(cuda_device):
    dev = cuda_device
    w = synth.WORKLOADS["llama2_layer_32k"].replace(P=3, L=4000, C=50, B=500, M=50, seed=5)
    K, V = synth.make_kv(w, device=dev)
    st, _, _, _ = _state(w, dev, K)
    q = synth.make_queries(w, device=dev)
    ref = st.step(q, K, V).clone()
    ref_sel = st.sel_idx.clone()
    st.enable_cache(1)
    out = st.step(q, K, V, step_no=0)
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(st.sel_idx, ref_sel)
    with pytest.raises(ValueError):
        st.step(q, K, V)
