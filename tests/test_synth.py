"""The seeded workload generator: shapes, value ranges, reproducibility."""
import numpy as np
import torch

from semantic_cluster_recall_b200 import synth


def test_workload_table():
    w = synth.WORKLOADS
    assert [w[k].name for k in synth.WORKLOAD_ORDER] == synth.WORKLOAD_ORDER
    c2 = w["llama2_layer_32k"]
    assert (c2.P, c2.L, c2.C, c2.T, c2.B, c2.S, c2.W, c2.N) == (32, 32768, 400, 10, 1024, 16, 64,
                                                                 32688)
    c4 = w["llama2_32layer_decode"]
    assert c4.P == 4096 and c4.L_cap == 32768 + 256 and c4.tail_cap == 320
    c5 = w["long_128k"]
    assert (c5.P, c5.L, c5.C, c5.T, c5.B, c5.W, c5.G) == (32, 131072, 1600, 8, 2048, 128, 4)


def test_mixture_keys_have_stated_norms_and_dtype():
    w = synth.WORKLOADS["tiny_f32"]
    K, V = synth.make_kv(w)
    assert K.shape == (1, 2048, 128) and K.dtype == torch.float32
    n = K.norm(dim=-1)
    assert float(n.min()) >= 0.5 - 1e-5 and float(n.max()) <= 2.0 + 1e-5
    assert abs(float(V.std()) - 1.0) < 0.02
    wb = synth.WORKLOADS["llama2_layer_32k"].replace(P=2, L=1024)
    Kb, _ = synth.make_kv(wb)
    assert Kb.dtype == torch.bfloat16


def test_problems_regenerate_alone_with_identical_bits():
    w = synth.WORKLOADS["llama3_gqa_32k"].replace(P=5, L=512)
    K, V = synth.make_kv(w)
    K3, V3 = synth.make_kv(w, problems=[3])
    assert torch.equal(K[3], K3[0]) and torch.equal(V[3], V3[0])
    q = synth.make_queries(w, step=2)
    q3 = synth.make_queries(w, step=2, problems=[3])
    assert torch.equal(q[3], q3[0]) and q.shape == (5, 4, 128)
    assert not torch.equal(q, synth.make_queries(w, step=3))


def test_keys_cluster_around_mixture_directions():
    # with small noise each key is close to one of its problem's directions
    w = synth.WORKLOADS["tiny_f32"].replace(sigma=0.01)
    K, _ = synth.make_kv(w)
    dirs = synth.directions(w, 0, "cpu")
    cos = (K[0] / K[0].norm(dim=-1, keepdim=True)) @ dirs.T
    assert float(cos.max(dim=1).values.min()) > 0.9


def test_random_labels_range_and_skew():
    lab = synth.random_labels(2, 5000, 50, seed=1, skew=1.2).numpy()
    assert lab.min() >= 0 and lab.max() < 50
    cnt = np.bincount(lab[0], minlength=50)
    assert cnt[0] > cnt[-1]


def test_correlated_queries_drift_with_rho():
    w = synth.WORKLOADS["llama2_layer_32k"].replace(P=4, L=256)
    dirs = synth.directions_all(w, "cpu")
    for rho in (0.0, 0.9, 0.99):
        q = synth.correlated_queries(w, dirs, 6, rho).float()
        assert q.shape == (6, 4, 1, 128)
        cos = torch.nn.functional.cosine_similarity(q[1:], q[:-1], dim=-1)
        assert abs(cos.mean().item() - rho) < 0.05
        # norms carry over from the first query
        n = torch.linalg.vector_norm(q, dim=-1)
        assert torch.allclose(n, n[:1].expand_as(n), rtol=2e-2)
    q1 = synth.correlated_queries(w, dirs, 3, 0.5)
    q2 = synth.correlated_queries(w, dirs, 3, 0.5)
    assert torch.equal(q1, q2)
