"""The 32-layer decode loop at full size (4096 problems, 69 GB of K/V).

Prefill clustering of every (layer, batch, head), then 256 decode steps that
each append one token and run the fused selection + sparse decode. The tail
holds the last W = 64 prompt tokens and grows by one per step; when an append
fills it to 320 tokens (at step 256), its oldest 256 tokens are clustered on
their own into 4 more clusters (10 rounds) and appended to the cluster
metadata ("III.B Clustering in the Semantic Space": generated tokens are
clustered alone into four new centroids every so many steps), before that
step's selection.

Checks: the incremental clustering of sampled problems against the oracle
(first divergent round only at near-ties), index invariants of the appended
metadata on every problem, and the final step teacher-forced: the sampled
problems get the oracle's metadata (prefill + incremental) and their
selection and attention are compared with the oracle's, in the same P = 4096
launch.
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


def _cluster_one(K, p, tb, te, C, iters, dev, dtype):
    """ckv_cluster on problem p alone (a one-problem view), fresh metadata."""
    n = te - tb
    cent = torch.zeros((1, C, 128), device=dev)
    hat = torch.zeros((1, C, 128), dtype=dtype, device=dev)
    lp = torch.zeros_like(hat)
    lab = torch.zeros((1, n), dtype=torch.int32, device=dev)
    sz = torch.zeros((1, C), dtype=torch.int32, device=dev)
    off = torch.zeros((1, C + 1), dtype=torch.int32, device=dev)
    perm = torch.zeros((1, n), dtype=torch.int32, device=dev)
    ws = ckv.workspace(ckv.ckv_cluster_workspace_bytes(1, n, C), dev)
    ckv.ckv_cluster(K[p:p + 1], K.stride(0), tb, te, C, iters, 0, 0, C, n, cent, hat, lp, lab,
                    sz, off, perm, ws, P=1)
    torch.cuda.synchronize()
    return lab[0].cpu().numpy(), cent[0].cpu().numpy(), off[0].cpu().numpy(), perm[0].cpu().numpy()


def test_decode_loop_with_incremental_clustering(cuda_device):
    dev = cuda_device
    w = synth.WORKLOADS["llama2_32layer_decode"]
    P, d, C, B = w.P, w.d, w.C, w.B
    tb, te = w.S, w.L - w.W
    N = te - tb
    n_inc = w.tail_cap - w.W            # 256 tokens clustered incrementally
    C_cap = C + w.inc_C
    perm_cap = N + n_inc
    K, V = synth.make_kv(w, device=dev)
    dirs = synth.directions_all(w, dev)
    st = ClusterRecall(P, w.G, d, w.torch_dtype, w.L_cap, w.S, B, C_cap, perm_cap, w.tail_cap,
                       dev)
    st.prefill(K, w.L, w.W, C, w.T)
    new_k = torch.empty((P, d), dtype=w.torch_dtype, device=dev)
    new_v = torch.empty_like(new_k)
    for step in range(1, w.steps + 1):
        pos = w.L + step - 1              # the generated token of this step
        new_k.copy_(K[:, pos])
        new_v.copy_(V[:, pos])
        st.append(K, V, new_k, new_v)
        if w.W + step == w.tail_cap:     # the tail is full: cluster its oldest tokens
            st.incremental(K, n_inc, w.inc_C, w.inc_T)
        q = synth.make_queries_batched(w, dirs, step)
        st.step(q, K, V)
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    assert st.C_used == C_cap and st.n_clustered == perm_cap
    te_final = w.L + w.steps
    inc_b, inc_e = te, te + n_inc
    assert (st.tail_begin.cpu().numpy() == inc_e).all()
    assert (st.tail_end.cpu().numpy() == te_final).all()
    cnt = st.sel_cnt.cpu().numpy()
    assert (cnt == min(B, perm_cap)).all()

    # index invariants of the appended clusters, every problem
    off = st.offsets.cpu().numpy()
    perm = st.perm.cpu().numpy()
    lab = st.labels.cpu().numpy()
    for p in range(P):
        o = off[p, C:C_cap + 1]
        assert o[0] == N and o[-1] == perm_cap and np.all(np.diff(o) >= 0)
        seg = perm[p, N:perm_cap]
        assert np.array_equal(np.sort(seg), np.arange(inc_b, inc_e))
        for c in range(w.inc_C):
            part = perm[p, o[c]:o[c + 1]]
            assert np.all(np.diff(part) > 0) and np.all(lab[p, part - inc_b + N] == C + c)

    # incremental clustering of sampled problems vs the oracle
    rng = np.random.default_rng(7)
    sampled = [int(x) for x in rng.choice(P, 4, replace=False)]
    for p in sampled:
        kh = f32np(K[p, inc_b:inc_e])
        r = oracle.kmeans(kh, w.inc_C, w.inc_T, "bf16", tok_begin=inc_b, perm_base=N,
                          history=True)
        got = lab[p, N:perm_cap] - C
        if not np.array_equal(got, r["labels"]):
            for t in range(1, w.inc_T + 1):  # first divergent round: near-ties only
                gl, _, _, _ = _cluster_one(K, p, inc_b, inc_e, w.inc_C, t, dev, w.torch_dtype)
                rt = oracle.kmeans(kh, w.inc_C, t, "bf16", tok_begin=inc_b, history=True)
                if not np.array_equal(gl, rt["labels"]):
                    bad = (gl != rt["labels"]) & (rt["gap_hist"][t - 1] >= GAP_EXEMPT)
                    assert not bad.any(), f"p={p} round {t}"
                    break
        else:
            assert np.array_equal(off[p, C:C_cap + 1], r["offsets"])
            assert np.array_equal(perm[p, N:perm_cap], r["perm"])
            err = centroid_rel_err(st.centroids[p, C:C_cap].cpu().numpy(), r["mu"])
            assert err.max() <= CENT_REL_L2

    # final step teacher-forced: oracle metadata for the sampled problems
    def oracle_meta(p):
        pre = oracle.kmeans(f32np(K[p, tb:te]), C, w.T, "bf16", tok_begin=tb)
        inc = oracle.kmeans(f32np(K[p, inc_b:inc_e]), w.inc_C, w.inc_T, "bf16",
                            tok_begin=inc_b, perm_base=N)
        mu = np.concatenate([pre["mu"], inc["mu"]])
        offs = np.concatenate([pre["offsets"][:-1], inc["offsets"]]).astype(np.int32)
        pm = np.concatenate([pre["perm"], inc["perm"]]).astype(np.int32)
        return p, mu, offs, pm

    metas = oracle.map_problems(oracle_meta, sampled)
    for p, mu, offs, pm in metas:
        st.centroids_lp[p] = torch.from_numpy(oracle.round_to(mu, "bf16").astype(np.float32)).to(
            w.torch_dtype)
        st.offsets[p] = torch.from_numpy(offs)
        st.perm[p] = torch.from_numpy(pm)
    q = synth.make_queries_batched(w, dirs, w.steps)
    out = st.step(q, K, V).cpu().numpy()
    torch.cuda.synchronize()
    assert ckv.ckv_device_error() == 0
    qh = f32np(q)
    sel_g = st.sel_idx.cpu().numpy()
    for p, mu, offs, pm in metas:
        s = oracle.score(qh[p], oracle.round_to(mu, "bf16"))
        sel, c = oracle.select(s, offs, pm, B)
        assert st.sel_cnt[p].item() == c and np.array_equal(sel_g[p, :c], sel)
        rows = oracle.attended_rows(w.S, sel, inc_e, te_final)
        ref = oracle.attend(qh[p], f32np(K[p]), f32np(V[p]), rows, 1 / math.sqrt(d))
        assert np.abs(out[p] - ref).max() <= OUT_MAX_ABS
