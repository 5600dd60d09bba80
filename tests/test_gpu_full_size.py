"""Parity at the workloads' full sizes, in the launch configurations the
benchmark times.

The inputs are generated on the device (same generator as everywhere), and
host copies of the problems the oracle needs are taken from those tensors.
Per workload:
  * assign: the oracle's strided seeds (cheap, all problems) feed ckv_assign
    over every problem; sampled tokens of sampled problems are compared with
    the oracle's argmax (labels equal except near-ties < 1e-4);
  * index, update: seeded labels feed both sides, every problem is compared
    (index bit-exact, sizes exact, centroids within 1e-3 relative L2);
  * selection + sparse decode (fused step): the oracle's centroids and index
    feed both sides, every problem is compared (selection bit-exact,
    attention within 2e-3);
  * round 1 of ckv_cluster on a sampled problem equals the oracle's round 1
    except near-ties; the full clustering run satisfies the index invariants
    on every problem.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from semantic_cluster_recall_b200 import ckv, synth
from semantic_cluster_recall_b200.pipeline import ClusterRecall

from helpers import CENT_REL_L2, GAP_EXEMPT, OUT_MAX_ABS, centroid_rel_err, f32np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLED_TOKENS = 2048


def _index_invariants(st, w, n_tok, tb, P):
    off = st.offsets[:, :w.C + 1].cpu().numpy()
    perm = st.perm[:, :n_tok].cpu().numpy()
    lab = st.labels[:, :n_tok].cpu().numpy()
    sizes = st.sizes[:, :w.C].cpu().numpy()
    for p in range(P):
        assert off[p, 0] == 0 and off[p, -1] == n_tok
        assert np.all(np.diff(off[p]) == sizes[p])
        assert lab[p].min() >= 0 and lab[p].max() < w.C
        assert np.array_equal(np.bincount(lab[p], minlength=w.C), sizes[p])
        assert np.array_equal(np.sort(perm[p]), np.arange(tb, tb + n_tok))
        for c in range(w.C):
            seg = perm[p, off[p, c]:off[p, c + 1]]
            assert np.all(np.diff(seg) > 0) and np.all(lab[p, seg - tb] == c)


@pytest.mark.parametrize("name", ["llama2_layer_32k", "llama3_gqa_32k", "long_128k"])
def test_full_size_workload(cuda_device, name):
    dev = cuda_device
    w = synth.WORKLOADS[name]
    P, C, d = w.P, w.C, w.d
    tb, te = w.S, w.L - w.W
    n = te - tb
    K, V = synth.make_kv(w, device=dev)
    q = synth.make_queries(w, device=dev)
    rng = np.random.default_rng(w.seed)

    # ---- end-to-end clustering (the benchmark's call) + invariants ----
    st = ClusterRecall(P, w.G, d, w.torch_dtype, w.L_cap, w.S, w.B, C, n, w.W, dev)
    st.prefill(K, w.L, w.W, C, w.T)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    _index_invariants(st, w, n, tb, P)

    # ---- round 1 of ckv_cluster on a sampled problem vs the oracle ----
    p1 = int(rng.integers(P))
    st1 = ClusterRecall(P, w.G, d, w.torch_dtype, w.L_cap, w.S, w.B, C, n, w.W, dev)
    st1.prefill(K, w.L, w.W, C, 1)
    Kh1 = f32np(K[p1, tb:te])
    r1 = oracle.kmeans(Kh1, C, 1, w.dtype, tok_begin=tb, history=True)
    lab1 = st1.labels[p1, :n].cpu().numpy()
    bad = (lab1 != r1["labels"]) & (r1["gap_hist"][0] >= GAP_EXEMPT)
    assert not bad.any(), f"round 1: {bad.sum()} non-tie label differences"
    del st1

    # ---- assign, teacher-forced with the oracle's seeds, sampled tokens ----
    hat = torch.zeros((P, C, d), dtype=w.torch_dtype, device=dev)
    seeds = {}
    for p in range(P):
        _, mh = oracle.init(f32np(K[p, tb:te]), C, w.dtype)
        seeds[p] = mh
        hat[p] = torch.from_numpy(mh.astype(np.float32)).to(w.torch_dtype)
    labels = torch.full((P, n), -1, dtype=torch.int32, device=dev)
    ckv.ckv_assign(K, K.stride(0), tb, te, hat, C, 0, C, labels, 0, n)
    torch.cuda.synchronize()
    lab = labels.cpu().numpy()
    for p in rng.choice(P, 4, replace=False):
        toks = np.sort(rng.choice(n, SAMPLED_TOKENS, replace=False))
        kh = f32np(K[p, tb:te])[toks]
        ref, gap = oracle.assign(kh, seeds[p])
        bad = (lab[p, toks] != ref) & (gap >= GAP_EXEMPT)
        assert not bad.any(), f"assign p={p}: {bad.sum()} non-tie differences"

    # ---- index + update from seeded labels, every problem ----
    lab_in = synth.random_labels(P, n, C, seed=w.seed, skew=0.5, device=dev)
    offsets = torch.full((P, C + 1), -1, dtype=torch.int32, device=dev)
    perm = torch.full((P, n), -1, dtype=torch.int32, device=dev)
    ws = ckv.workspace(ckv.ckv_index_workspace_bytes(P, n, C), dev)
    ckv.ckv_index(lab_in, P, tb, te, C, 0, C, 0, n, offsets, perm, ws)
    cent = torch.zeros((P, C, d), device=dev)
    hat2 = torch.zeros((P, C, d), dtype=w.torch_dtype, device=dev)
    lp = torch.zeros_like(hat2)
    sizes = torch.zeros((P, C), dtype=torch.int32, device=dev)
    ckv.ckv_update(K, K.stride(0), tb, te, C, 0, C, offsets, perm, n, cent, hat2, lp, sizes)
    torch.cuda.synchronize()
    lab_h = lab_in.cpu().numpy()
    off_h, perm_h = offsets.cpu().numpy(), perm.cpu().numpy()
    cent_h, sizes_h = cent.cpu().numpy(), sizes.cpu().numpy()
    mu_or = np.zeros((P, C, d))
    off_or = np.zeros((P, C + 1), np.int32)
    perm_or = np.zeros((P, n), np.int32)

    def per_problem(p):
        kh = f32np(K[p, tb:te])
        o, pm = oracle.index(lab_h[p], C, tb, 0)
        mu, _, sz = oracle.update(kh, lab_h[p], np.zeros((C, d)), np.zeros((C, d)), w.dtype)
        return p, o, pm, mu, sz

    for p, o, pm, mu, sz in oracle.map_problems(per_problem, list(range(P))):
        assert np.array_equal(off_h[p], o) and np.array_equal(perm_h[p], pm), f"index p={p}"
        assert np.array_equal(sizes_h[p], sz)
        nz = sz > 0
        assert centroid_rel_err(cent_h[p][nz], mu[nz]).max() <= CENT_REL_L2, f"update p={p}"
        mu_or[p], off_or[p], perm_or[p] = mu, o, pm

    # ---- fused selection + sparse decode from the oracle's metadata ----
    mode = w.dtype
    st2 = ClusterRecall(P, w.G, d, w.torch_dtype, w.L_cap, w.S, w.B, C, n, w.W, dev)
    st2.centroids_lp.copy_(torch.from_numpy(oracle.round_to(mu_or, mode).astype(np.float32)))
    st2.offsets.copy_(torch.from_numpy(off_or))
    st2.perm.copy_(torch.from_numpy(perm_or))
    st2.n_clusters.fill_(C)
    st2.tail_begin.fill_(te)
    st2.tail_end.fill_(w.L)
    out = st2.step(q, K, V)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    sel_g, cnt_g, out_g = st2.sel_idx.cpu().numpy(), st2.sel_cnt.cpu().numpy(), out.cpu().numpy()
    qh = f32np(q)
    lp_or = oracle.round_to(mu_or, mode).astype(np.float32)

    def decode_ref(p):
        s = oracle.score(qh[p], lp_or[p])
        sel, cnt = oracle.select(s, off_or[p], perm_or[p], w.B)
        rows = oracle.attended_rows(w.S, sel, te, w.L)
        att = oracle.attend(qh[p], f32np(K[p]), f32np(V[p]), rows, 1 / math.sqrt(d))
        return p, sel, cnt, att

    for p, sel, cnt, att in oracle.map_problems(decode_ref, list(range(P))):
        assert cnt_g[p] == cnt and np.array_equal(sel_g[p, :cnt], sel), f"select p={p}"
        assert np.abs(out_g[p] - att).max() <= OUT_MAX_ABS, f"decode p={p}"


def test_tiny_f32_end_to_end(cuda_device):
    # the fp32 workload is small enough for a full end-to-end comparison:
    # labels must agree up to the first round with a near-tie difference
    dev = cuda_device
    w = synth.WORKLOADS["tiny_f32"]
    K, V = synth.make_kv(w)
    Kh = f32np(K)
    Kd = K.to(dev)
    tb, te = w.S, w.L - w.W
    n = te - tb
    for t in range(1, w.T + 1):
        st = ClusterRecall(w.P, w.G, w.d, torch.float32, w.L_cap, w.S, w.B, w.C, n, w.W, dev)
        st.prefill(Kd, w.L, w.W, w.C, t)
        r = oracle.kmeans(Kh[0, tb:te], w.C, t, "f32", tok_begin=tb, history=True)
        lab = st.labels[0, :n].cpu().numpy()
        if not np.array_equal(lab, r["labels"]):
            bad = (lab != r["labels"]) & (r["gap_hist"][t - 1] >= GAP_EXEMPT)
            assert not bad.any()
            break
        assert centroid_rel_err(f32np(st.centroids[0, :w.C]), r["mu"]).max() <= CENT_REL_L2
        assert np.array_equal(st.perm[0, :n].cpu().numpy(), r["perm"])


@pytest.mark.parametrize("metric", ["ip", "l2"])
def test_full_size_assign_by_similarity(cuda_device, metric):
    # the bench's assign_by_similarity launches (seeding + one assignment round
    # of the bench workload under the distance ablation): seeds bit-exact on
    # every problem, sampled tokens of sampled problems against the oracle
    dev = cuda_device
    w = synth.WORKLOADS["llama2_layer_32k"]
    P, C, d = w.P, w.C, w.d
    tb, te = w.S, w.L - w.W
    n = te - tb
    K, _ = synth.make_kv(w, device=dev, rows=w.L)
    cent = torch.zeros((P, C, d), device=dev)
    hat = torch.zeros((P, C, d), dtype=w.torch_dtype, device=dev)
    lp = torch.zeros_like(hat)
    bias = torch.zeros((P, C), device=dev)
    labels = torch.full((P, n), -1, dtype=torch.int32, device=dev)
    ckv.ckv_init_centroids_ex(K, K.stride(0), tb, te, C, 0, C, cent, hat, lp, metric=metric,
                              bias=bias)
    ckv.ckv_assign_ex(K, K.stride(0), tb, te, hat, C, 0, C, labels, 0, n,
                      bias=bias if metric == "l2" else None)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    rng = np.random.default_rng(w.seed + 7)
    lab = labels.cpu().numpy()
    hat_h = hat.float().cpu().numpy().astype(np.float64)
    for p in rng.choice(P, 3, replace=False):
        kh = f32np(K[p, tb:te])
        _, mh = oracle.init(kh, C, w.dtype, metric=metric)
        assert np.array_equal(hat_h[p], mh)
        toks = np.sort(rng.choice(n, SAMPLED_TOKENS, replace=False))
        ref, gap = oracle.assign(kh[toks], mh, metric=metric)
        bad = (lab[p, toks] != ref) & (gap >= GAP_EXEMPT)
        assert not bad.any(), f"{metric} p={p}: {bad.sum()} non-tie differences"
