"""Background clustering of generated tokens, overlapped with decode steps.

The oldest tail tokens that the incremental clustering takes exist well
before the tail is full, so the clustering can start early on a side stream
(low priority, the tensor-core assignment held to a few SMs) while the main
stream keeps appending and decoding, and be published when the tail fills
("IV.B Semantic Clustering": clustering is launched asynchronously and
overlaps other inference work; "III.B": generated tokens are clustered on
their own into four new centroids).

Two runs of the same decode loop, one clustering synchronously when the tail
fills and one in the background, must give bit-identical outputs at every
step (the steps read only published clusters, and the kernels are
deterministic) and bit-identical metadata at the end. The synchronous run is
itself checked against the oracle elsewhere (the 32-layer decode loop test).

Prefill from host memory overlaps the upload of one group of problems with
the clustering of the previous ones; it must give the same metadata as the
one-call clustering of the same keys already on the device.
"""
import numpy as np
import pytest
import torch

from semantic_cluster_recall_b200 import ckv, synth
from semantic_cluster_recall_b200.pipeline import ClusterRecall

pytestmark = pytest.mark.gpu

W_SMALL = synth.WORKLOADS["llama2_32layer_decode"].replace(
    P=48, L=2048, C=25, B=256, M=25, W=32, tail_cap=96, steps=72, layers=1, batch=1,
    heads_kv=48)


def _loop(w, K, V, dirs, dev, background: bool):
    n_inc = w.tail_cap - w.W
    tb, te = w.S, w.L - w.W
    N = te - tb
    main = torch.cuda.Stream(device=dev, priority=-1)
    side = torch.cuda.Stream(device=dev, priority=0)
    st = ClusterRecall(w.P, w.G, w.d, w.torch_dtype, w.L_cap, w.S, w.B, w.C + w.inc_C,
                       N + n_inc, w.tail_cap, dev, stream=main)
    outs = []
    with torch.cuda.stream(main):
        st.prefill(K, w.L, w.W, w.C, w.T)
        new_k = torch.empty((w.P, w.d), dtype=w.torch_dtype, device=dev)
        new_v = torch.empty_like(new_k)
        for step in range(1, w.steps + 1):
            pos = w.L + step - 1
            new_k.copy_(K[:, pos])
            new_v.copy_(V[:, pos])
            st.append(K, V, new_k, new_v)
            if background and w.W + step == n_inc:   # the oldest n_inc tail tokens exist
                st.incremental_begin(K, n_inc, w.inc_C, w.inc_T, side, max_sms=8)
            if w.W + step == w.tail_cap:              # the tail is full
                if background:
                    st.incremental_commit()
                else:
                    st.incremental(K, n_inc, w.inc_C, w.inc_T)
            q = synth.make_queries_batched(w, dirs, step)
            out = st.step(q, K, V)
            outs.append((out.clone(), st.sel_idx.clone(), st.sel_cnt.clone()))
    torch.cuda.synchronize()
    return st, outs


def test_background_incremental_clustering_is_identical(cuda_device):
    dev = cuda_device
    w = W_SMALL
    K, V = synth.make_kv(w, device=dev)
    dirs = synth.directions_all(w, dev)
    st_a, out_a = _loop(w, K, V, dirs, dev, background=False)
    st_b, out_b = _loop(w, K, V, dirs, dev, background=True)
    assert ckv.ckv_device_error() == 0
    assert len(out_a) == len(out_b) == w.steps
    for i, ((oa, sa, ca), (ob, sb, cb)) in enumerate(zip(out_a, out_b)):
        assert torch.equal(ca, cb), f"step {i + 1}: counts"
        assert torch.equal(sa, sb), f"step {i + 1}: selection"
        assert torch.equal(oa, ob), f"step {i + 1}: output"
    for name in ("n_clusters", "tail_begin", "tail_end", "offsets", "perm", "labels", "sizes",
                 "centroids", "centroids_hat", "centroids_lp"):
        assert torch.equal(getattr(st_a, name), getattr(st_b, name)), name
    assert (st_a.C_used, st_a.n_clustered, st_a.tail_lo) == \
        (st_b.C_used, st_b.n_clustered, st_b.tail_lo)
    # the appended clusters are a valid index of the clustered tail tokens
    n_inc = w.tail_cap - w.W
    N = w.N
    off = st_b.offsets.cpu().numpy()[:, w.C:w.C + w.inc_C + 1]
    perm = st_b.perm.cpu().numpy()[:, N:N + n_inc]
    inc_b = w.L - w.W
    for p in range(w.P):
        assert off[p, 0] == N and off[p, -1] == N + n_inc
        assert np.array_equal(np.sort(perm[p]), np.arange(inc_b, inc_b + n_inc))


def test_background_clustering_guards(cuda_device):
    dev = cuda_device
    w = W_SMALL.replace(P=2)
    K, _ = synth.make_kv(w, device=dev)
    st = ClusterRecall(w.P, w.G, w.d, w.torch_dtype, w.L_cap, w.S, w.B, w.C + w.inc_C,
                       w.N + 64, w.tail_cap, dev)
    st.prefill(K, w.L, w.W, w.C, 2)
    with pytest.raises(RuntimeError):
        st.incremental_commit()
    side = torch.cuda.Stream(device=dev)
    st.incremental_begin(K, 32, w.inc_C, 2, side, max_sms=4)
    with pytest.raises(RuntimeError):
        st.incremental_begin(K, 32, w.inc_C, 2, side)
    st.incremental_commit()
    torch.cuda.synchronize()
    assert int(st.n_clusters[0]) == w.C + w.inc_C
    assert ckv.ckv_device_error() == 0


def test_prefill_from_host_equals_prefill(cuda_device):
    # uploading in groups on a copy stream, each group clustered as it lands,
    # gives the same metadata as clustering the device copy in one call
    dev = cuda_device
    w = W_SMALL.replace(P=10)
    K, V = synth.make_kv(w, device=dev)
    Kh = K.cpu().pin_memory()
    Vh = V.cpu().pin_memory()
    tb, te = w.S, w.L - w.W
    n = te - tb
    a = ClusterRecall(w.P, w.G, w.d, w.torch_dtype, w.L_cap, w.S, w.B, w.C, n, w.W, dev)
    a.prefill(K, w.L, w.W, w.C, w.T)
    Kd = torch.zeros_like(K)
    Vd = torch.zeros_like(V)
    main = torch.cuda.Stream(device=dev)
    b = ClusterRecall(w.P, w.G, w.d, w.torch_dtype, w.L_cap, w.S, w.B, w.C, n, w.W, dev,
                      stream=main)
    with torch.cuda.stream(main):
        b.prefill_from_host(Kh, Vh, Kd, Vd, w.L, w.W, w.C, w.T, torch.cuda.Stream(device=dev),
                            groups=3)
    torch.cuda.synchronize()
    assert torch.equal(Kd[:, :w.L], K[:, :w.L]) and torch.equal(Vd[:, :w.L], V[:, :w.L])
    for name in ("labels", "sizes", "offsets", "perm", "centroids", "centroids_hat",
                 "centroids_lp", "n_clusters", "tail_begin", "tail_end"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    q = synth.make_queries(w, device=dev)
    out_a = a.step(q, K, V)
    with torch.cuda.stream(main):
        out_b = b.step(q, Kd, Vd)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
