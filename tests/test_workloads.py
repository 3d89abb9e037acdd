"""The seeded input generators: shapes, determinism and the stated recipe."""
import numpy as np

from sparse_attention_indexer_05_b200 import workloads as W


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, -2.5, 1.0 + 2**-9, 3.0e38], np.float32)
    got = W.bf16_to_f32(W.bf16_bits(x))
    want = np.array([1.0, 1.0, 1.0 + 2**-6, -2.5, 1.0, 2.9983e38], np.float32)
    assert np.array_equal(got[:5], want[:5])
    assert abs(got[5] / 3.0e38 - 1) < 2**-8


def test_keys_planted_fraction_and_direction():
    L, d = 4000, 128
    k = W.bf16_to_f32(W.keys(L, d, 0.01, seed=1)).astype(np.float64)
    u = W.rng_for(1, 4, 0).standard_normal(d)
    u /= np.linalg.norm(u)
    proj = k @ u
    planted = proj > 20
    assert planted.sum() == 40                       # exactly floor(0.01 L)
    assert abs(proj[planted].mean() - 4 * np.sqrt(d)) < 0.5
    assert abs(proj[~planted].std() - 1.0) < 0.1


def test_queries_ar1_correlation_and_determinism():
    q = W.bf16_to_f32(W.queries_ar1(3000, 2, 16, 0.95, seed=2)).astype(np.float64)
    x = q.reshape(3000, -1)
    r = (x[1:] * x[:-1]).mean() / (x * x).mean()
    assert abs(r - 0.95) < 0.02
    assert abs(x.std() - 1.0) < 0.1
    q2 = W.queries_ar1(3000, 2, 16, 0.95, seed=2)
    assert np.array_equal(W.bf16_bits(q.astype(np.float32)), q2)


def test_weights_range_and_configs_shapes():
    w = W.weights(100, 64, seed=0)
    assert w.min() >= 0 and w.max() < 1 / 64
    P = W.prefill([33, 17], H=4, d=32, topk=8)
    assert P.q.shape == (50, 4, 32) and P.k.shape == (50, 32) and P.w.shape == (50, 4)
    assert P.cu_seqlens.tolist() == [0, 33, 50]
    D = W.decode(B=3, n=64, G=2, H=4, d=32, topk=8)
    assert D.q.shape == (3, 2, 4, 32) and D.kcache.shape == (3, 64, 32) and D.kv_len.tolist() == [64] * 3
    S = W.small_fp32()
    assert S.q.dtype == np.float32 and S.q.shape == (2048, 4, 64)
    assert abs(S.q.std() - 1 / 8) < 0.005


def test_empty_request_in_a_pack():
    P = W.prefill([5, 0, 3], H=2, d=8, topk=2)
    assert P.q.shape == (8, 2, 8) and P.cu_seqlens.tolist() == [0, 5, 5, 8]
