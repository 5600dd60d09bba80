"""Parity of the fused decode step (ckv_select_decode) with the oracle.

The fused kernel must give the same selection as the oracle bit for bit
(sel_cnt and sel_idx, given the oracle's centroids and index) and attention
within 2e-3 max-abs of the oracle's double attention over that selection.
"""
import numpy as np
import pytest
import torch

import oracle
from semantic_cluster_recall_b200 import ckv, synth

from helpers import OUT_MAX_ABS, mode_of, to_dev

pytestmark = pytest.mark.gpu


def _case(dev, dtype, P, G, C, n, budget, L, S, tails, seed, ties=False, n_clusters=None,
          skew=0.8, q_scale=1.0, all_equal=False, singletons=False):
    rng = np.random.default_rng(seed)
    mode = mode_of(dtype)
    d = 128
    tb0 = S
    C_cap, perm_cap = C + 3, n + 5
    lab = synth.random_labels(P, n, C, seed=seed, skew=skew).numpy()
    if singletons:  # every token its own cluster
        assert C == n
        lab = np.stack([rng.permutation(n) for _ in range(P)]).astype(np.int32)
    mu = rng.standard_normal((P, C, d)) * 0.3
    if ties:
        mu[:, 1::3] = mu[:, 0:-1:3][:, :mu[:, 1::3].shape[1]]
    if all_equal:  # one score for every cluster: the id order decides alone
        mu[:] = mu[:, :1]
    mu_lp = oracle.round_to(mu, mode).astype(np.float32)
    q = oracle.round_to(rng.standard_normal((P, G, d)) * q_scale, mode).astype(np.float32)
    K = oracle.round_to(rng.standard_normal((P, L, d)) * 0.5, mode).astype(np.float32)
    V = oracle.round_to(rng.standard_normal((P, L, d)), mode).astype(np.float32)
    ncl = np.full(P, C, np.int32) if n_clusters is None else np.asarray(n_clusters, np.int32)
    lp_np = np.zeros((P, C_cap, d), np.float32)
    lp_np[:, :C] = mu_lp
    off_np = np.zeros((P, C_cap + 1), np.int32)
    perm_np = np.full((P, perm_cap), -1, np.int32)
    tb = np.array([t[0] for t in tails], np.int32)
    te = np.array([t[1] for t in tails], np.int32)
    refs = []
    for p in range(P):
        o, pm = oracle.index(lab[p], C, tb0, 0)
        off_np[p, :C + 1] = o
        perm_np[p, :n] = pm
        s = oracle.score(q[p], mu_lp[p][:ncl[p]])
        sel, cnt = oracle.select(s, o[:ncl[p] + 1], pm, budget)
        rows = oracle.attended_rows(S, sel, tb[p], te[p])
        refs.append((sel, cnt, oracle.attend(q[p], K[p], V[p], rows, 1 / np.sqrt(d))))
    Kd, Vd = to_dev(K, dtype, dev), to_dev(V, dtype, dev)
    sel_d = torch.full((P, max(budget, 1)), -9, dtype=torch.int32, device=dev)
    cnt_d = torch.full((P,), -9, dtype=torch.int32, device=dev)
    out = torch.full((P, G, d), float("nan"), device=dev)
    max_tail = int((te - tb).max())
    args = dict(q=to_dev(q, dtype, dev), lp=to_dev(lp_np, dtype, dev),
                ncl=torch.from_numpy(ncl).to(dev), C_cap=C_cap,
                off=torch.from_numpy(off_np).to(dev), perm=torch.from_numpy(perm_np).to(dev),
                perm_cap=perm_cap, budget=budget, K=Kd, V=Vd, L=L, S=S,
                tb=torch.from_numpy(tb).to(dev), te=torch.from_numpy(te).to(dev),
                max_tail=max_tail)
    ckv.ckv_select_decode(args["q"], args["lp"], args["ncl"], C_cap, args["off"], args["perm"],
                          perm_cap, budget, sel_d, cnt_d, Kd, Vd, Kd.stride(0), L, S, args["tb"],
                          args["te"], max_tail, 1 / np.sqrt(d), out)
    torch.cuda.synchronize()
    return refs, sel_d.cpu().numpy(), cnt_d.cpu().numpy(), out.cpu().numpy(), args


def _check(refs, sel, cnt, out):
    for p, (r_sel, r_cnt, r_out) in enumerate(refs):
        assert cnt[p] == r_cnt, (p, cnt[p], r_cnt)
        assert np.array_equal(sel[p, :r_cnt], r_sel), f"problem {p}"
        err = np.abs(out[p] - r_out).max()
        assert err <= OUT_MAX_ABS, (p, err)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("G", [1, 2, 4])
@pytest.mark.parametrize("budget", [0, 1, 300, 1024, 5000])
def test_fused_step_matches_oracle(cuda_device, dtype, G, budget):
    P, L, S = 5, 5000, 16
    tails = [(4936, 5000), (4900, 5000), (4990, 4990), (4000, 4320), (4999, 5000)]
    refs, sel, cnt, out, _ = _case(cuda_device, dtype, P, G, C=400, n=3900, budget=budget, L=L,
                                   S=S, tails=tails, seed=budget * 7 + G)
    _check(refs, sel, cnt, out)
    assert ckv.ckv_device_error() == 0


def test_fused_step_ties_large_C_partial_counts_no_sinks(cuda_device):
    P, L, S = 3, 24000, 0
    tails = [(23000, 23100), (23500, 23500), (22000, 22300)]
    refs, sel, cnt, out, _ = _case(cuda_device, torch.bfloat16, P, 4, C=1604, n=20000,
                                   budget=2048, L=L, S=S, tails=tails, seed=5, ties=True,
                                   n_clusters=[1604, 1600, 17], q_scale=6.0)
    _check(refs, sel, cnt, out)
    assert ckv.ckv_device_error() == 0


@pytest.mark.parametrize("G,dtype", [(1, torch.bfloat16), (2, torch.bfloat16),
                                     (4, torch.bfloat16), (4, torch.float32)])
def test_fused_step_many_problems_single_cta_clusters(cuda_device, G, dtype):
    # enough problems that each cluster is a single CTA (the many-problem
    # instantiations with fewer rows in flight)
    P, L, S = 700, 1500, 4
    tails = [(1400, 1400 + (p % 64)) for p in range(P)]
    refs, sel, cnt, out, _ = _case(cuda_device, dtype, P, G, C=40, n=1300, budget=256,
                                   L=L, S=S, tails=tails, seed=11 + G)
    _check(refs, sel, cnt, out)
    assert ckv.ckv_device_error() == 0


def test_fused_step_equals_separate_calls(cuda_device):
    P, L, S = 6, 6000, 16
    tails = [(5936, 6000)] * P
    refs, sel, cnt, out, a = _case(cuda_device, torch.bfloat16, P, 4, C=400, n=5000,
                                   budget=1024, L=L, S=S, tails=tails, seed=3)
    dev = cuda_device
    sel2 = torch.full((P, 1024), -9, dtype=torch.int32, device=dev)
    cnt2 = torch.full((P,), -9, dtype=torch.int32, device=dev)
    ws = ckv.workspace(ckv.ckv_select_workspace_bytes(P, a["C_cap"]), dev)
    ckv.ckv_select(a["q"], a["lp"], a["ncl"], a["C_cap"], a["off"], a["perm"], a["perm_cap"],
                   1024, sel2, cnt2, ws)
    out2 = torch.empty((P, 4, 128), device=dev)
    wsd = ckv.workspace(ckv.ckv_decode_workspace_bytes(P, 4, 128, S + 1024 + 64), dev)
    ckv.ckv_sparse_decode(a["q"], a["K"], a["V"], a["K"].stride(0), L, S, a["tb"], a["te"], 64,
                          sel2, cnt2, 1024, 1 / np.sqrt(128), out2, wsd)
    torch.cuda.synchronize()
    assert np.array_equal(cnt2.cpu().numpy(), cnt)
    assert np.array_equal(sel2.cpu().numpy(), sel)
    assert np.abs(out2.cpu().numpy() - out).max() <= 1e-5


@pytest.mark.parametrize("budget", [1, 777, 3900])
def test_fused_step_all_scores_equal(cuda_device, budget):
    # identical centroids: the selection is decided by cluster id alone
    # (budget 3900 equals the clustered total exactly)
    P, L, S = 3, 5000, 16
    tails = [(4936, 5000)] * P
    refs, sel, cnt, out, _ = _case(cuda_device, torch.bfloat16, P, 2, C=400, n=3900,
                                   budget=budget, L=L, S=S, tails=tails, seed=21,
                                   all_equal=True)
    _check(refs, sel, cnt, out)
    assert ckv.ckv_device_error() == 0


@pytest.mark.parametrize("P,C", [(2, 4000), (600, 1100)])
def test_fused_step_singleton_clusters(cuda_device, P, C):
    # C = n: every cluster holds one token, so the budget selects 1024
    # clusters, the top-B tokens by q . k (the largest selected set); 600
    # problems make every problem a single CTA
    S = 4
    L = S + C + 64
    tails = [(S + C, S + C + (p % 50)) for p in range(P)]
    refs, sel, cnt, out, _ = _case(cuda_device, torch.bfloat16, P, 1, C=C, n=C,
                                   budget=1024, L=L, S=S, tails=tails, seed=23,
                                   singletons=True)
    _check(refs, sel, cnt, out)
    assert ckv.ckv_device_error() == 0
