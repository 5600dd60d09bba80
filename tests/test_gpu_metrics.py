"""Clustering under the paper's distance ablation: inner product and L2.

"III.B Clustering in the Semantic Space" of "ClusterKV: Manipulating LLM KV
Cache in Semantic Space for Recallable Compression" clusters by cosine
similarity and compares it with L2 and inner-product clustering. The CUDA
path runs both as the same kernels with a flag: the assignment copy is the
raw mean rounded to storage, and L2 subtracts half of its squared norm (an
fp32 bias per centroid) from every score in the argmax epilogue.

Parity, stage by stage as for cosine: seeding and update must give the
oracle's assignment copies bit for bit and the bias within fp32 rounding;
assignment from the oracle's copies must give the oracle's labels except at
near-ties (oracle top-2 gap < 1e-4 over the key norm); on planted blocks the
whole clustering must match the oracle's exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from semantic_cluster_recall_b200 import ckv, synth

from helpers import CENT_REL_L2, GAP_EXEMPT, f32np, mode_of, small_workload

pytestmark = pytest.mark.gpu

METRICS = ["ip", "l2"]
DTYPES = [torch.bfloat16, torch.float32]


def _half_sq_norm(m: np.ndarray) -> np.ndarray:
    return (0.5 * np.sum(m.astype(np.float64) ** 2, axis=-1)).astype(np.float32)


def _bufs(P, C_cap, dtype, dev):
    return (torch.zeros((P, C_cap, 128), device=dev),
            torch.zeros((P, C_cap, 128), dtype=dtype, device=dev),
            torch.zeros((P, C_cap, 128), dtype=dtype, device=dev),
            torch.full((P, C_cap), float("nan"), device=dev))


@pytest.mark.parametrize("metric", METRICS)
@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("C", [40, 300, 1100])
def test_seed_and_assign_match_oracle(cuda_device, metric, dtype, C):
    dev = cuda_device
    w = small_workload(dtype, P=3, L=6000, C=C, T=1)
    K, _ = synth.make_kv(w)
    Kd = K.to(dev)
    tb, te = w.S, w.L - w.W
    n = te - tb
    cbase, C_cap = 3, C + 5  # clusters at an offset inside the capacity
    cent, hat, lp, bias = _bufs(w.P, C_cap, dtype, dev)
    ckv.ckv_init_centroids_ex(Kd, Kd.stride(0), tb, te, C, cbase, C_cap, cent, hat, lp,
                              metric=metric, bias=bias)
    labels = torch.full((w.P, n), -1, dtype=torch.int32, device=dev)
    ckv.ckv_assign_ex(Kd, Kd.stride(0), tb, te, hat, C, cbase, C_cap, labels, 0, n,
                      bias=bias if metric == "l2" else None)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    Kh = f32np(K)
    for p in range(w.P):
        mu, mh = oracle.init(Kh[p, tb:te], C, mode_of(dtype), metric=metric)
        assert np.array_equal(f32np(hat[p, cbase:cbase + C]).astype(np.float64), mh)
        if metric == "l2":
            np.testing.assert_allclose(bias[p, cbase:cbase + C].cpu().numpy(), _half_sq_norm(mh),
                                       rtol=2e-7)
        ref, gap = oracle.assign(Kh[p, tb:te], mh, metric=metric)
        got = labels[p].cpu().numpy() - cbase
        bad = (got != ref) & (gap >= GAP_EXEMPT)
        assert not bad.any(), f"p={p}: {bad.sum()} non-tie differences"
        assert (got == ref).mean() > 0.99


@pytest.mark.parametrize("metric", METRICS)
@pytest.mark.parametrize("dtype", DTYPES)
def test_update_matches_oracle(cuda_device, metric, dtype):
    dev = cuda_device
    w = small_workload(dtype, P=3, L=5000, C=70, T=1)
    K, _ = synth.make_kv(w)
    Kd = K.to(dev)
    tb, te = w.S, w.L - w.W
    n, C = te - tb, w.C
    lab = synth.random_labels(w.P, n, C, seed=77, skew=0.6)
    lab[:, :] = torch.where(lab == 5, torch.full_like(lab, 6), lab)  # cluster 5 stays empty
    labd = lab.to(dev)
    offsets = torch.zeros((w.P, C + 1), dtype=torch.int32, device=dev)
    perm = torch.zeros((w.P, n), dtype=torch.int32, device=dev)
    ws = ckv.workspace(ckv.ckv_index_workspace_bytes(w.P, n, C), dev)
    ckv.ckv_index(labd, w.P, tb, te, C, 0, C, 0, n, offsets, perm, ws)
    cent, hat, lp, bias = _bufs(w.P, C, dtype, dev)
    sentinel = torch.full((128,), 0.25, dtype=dtype, device=dev)
    hat[:, 5] = sentinel
    bias[:, 5] = 1.5
    sizes = torch.zeros((w.P, C), dtype=torch.int32, device=dev)
    ckv.ckv_update_ex(Kd, Kd.stride(0), tb, te, C, 0, C, offsets, perm, n, cent, hat, lp, sizes,
                      metric=metric, bias=bias)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    Kh = f32np(K)
    mode = mode_of(dtype)
    for p in range(w.P):
        mu0 = np.zeros((C, 128))
        mu, mh, sz = oracle.update(Kh[p, tb:te], lab[p].numpy(), mu0, mu0, mode, metric=metric)
        assert np.array_equal(sizes[p].cpu().numpy(), sz) and sz[5] == 0
        live = sz > 0
        assert np.array_equal(f32np(hat[p])[live].astype(np.float64), mh[live])
        assert np.array_equal(f32np(lp[p])[live].astype(np.float64), oracle.round_to(mu, mode)[live])
        err = np.linalg.norm(f32np(cent[p])[live] - mu[live], axis=1) / \
            np.linalg.norm(mu[live], axis=1)
        assert err.max() <= CENT_REL_L2
        # the empty cluster keeps its previous copy and bias
        assert torch.equal(hat[p, 5], sentinel)
        if metric == "l2":
            b = bias[p].cpu().numpy()
            np.testing.assert_allclose(b[live], _half_sq_norm(mh[live]), rtol=2e-7)
            assert b[5] == 1.5


@pytest.mark.parametrize("metric", METRICS)
@pytest.mark.parametrize("dtype", DTYPES)
def test_whole_clustering_on_planted_blocks(cuda_device, metric, dtype):
    # well separated blocks: no near-ties, so every round must agree exactly
    dev = cuda_device
    w = small_workload(dtype, P=4, L=4000, C=48, T=5,
                       sigma=0.3 / np.sqrt(128)).replace(planted=True)
    K, _ = synth.make_kv(w)
    Kd = K.to(dev)
    tb, te = w.S, w.L - w.W
    n, C = te - tb, w.C
    cent, hat, lp, _ = _bufs(w.P, C, dtype, dev)
    labels = torch.zeros((w.P, n), dtype=torch.int32, device=dev)
    sizes = torch.zeros((w.P, C), dtype=torch.int32, device=dev)
    offsets = torch.zeros((w.P, C + 1), dtype=torch.int32, device=dev)
    perm = torch.zeros((w.P, n), dtype=torch.int32, device=dev)
    ws = ckv.workspace(ckv.ckv_cluster_ex_workspace_bytes(w.P, n, C, metric), dev)
    ckv.ckv_cluster_ex(Kd, Kd.stride(0), tb, te, C, w.T, 0, 0, C, n, cent, hat, lp, labels,
                       sizes, offsets, perm, ws, metric=metric)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    Kh = f32np(K)
    for p in range(w.P):
        r = oracle.kmeans(Kh[p, tb:te], C, w.T, mode_of(dtype), tok_begin=tb, metric=metric)
        assert np.array_equal(labels[p].cpu().numpy(), r["labels"]), p
        assert np.array_equal(offsets[p].cpu().numpy(), r["offsets"])
        assert np.array_equal(perm[p].cpu().numpy(), r["perm"])
        assert np.array_equal(f32np(hat[p]).astype(np.float64), r["muhat"])
        err = np.linalg.norm(f32np(cent[p]) - r["mu"], axis=1) / np.linalg.norm(r["mu"], axis=1)
        assert err.max() <= CENT_REL_L2


def test_cosine_through_the_ex_calls_is_unchanged(cuda_device):
    # ckv_cluster_ex with the cosine metric and ckv_cluster give the same bits
    dev = cuda_device
    w = small_workload(torch.bfloat16, P=2, L=5000, C=80, T=3)
    K, _ = synth.make_kv(w)
    Kd = K.to(dev)
    tb, te = w.S, w.L - w.W
    n, C = te - tb, w.C
    outs = []
    for use_ex in (False, True):
        cent, hat, lp, _ = _bufs(w.P, C, torch.bfloat16, dev)
        labels = torch.zeros((w.P, n), dtype=torch.int32, device=dev)
        sizes = torch.zeros((w.P, C), dtype=torch.int32, device=dev)
        offsets = torch.zeros((w.P, C + 1), dtype=torch.int32, device=dev)
        perm = torch.zeros((w.P, n), dtype=torch.int32, device=dev)
        ws = ckv.workspace(ckv.ckv_cluster_workspace_bytes(w.P, n, C), dev)
        args = (Kd, Kd.stride(0), tb, te, C, w.T, 0, 0, C, n, cent, hat, lp, labels, sizes,
                offsets, perm, ws)
        if use_ex:
            ckv.ckv_cluster_ex(*args, metric="cos")
        else:
            ckv.ckv_cluster(*args)
        torch.cuda.synchronize()
        outs.append((cent, hat, lp, labels, sizes, offsets, perm))
    for a, b in zip(*outs):
        assert torch.equal(a, b)
