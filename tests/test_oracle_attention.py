"""Pins of the oracle's paged attention and log2-sum-exp fold.

Split-KV paged decode attention with inline dequantisation (mistral.rs PR
"YaRN rope scaling, 4-bit F4 packed KV cache, ...", section 2, v1/v2
paged_attention) and partials folded by log2-sum-exp (FreeToken issue #568,
proposed solution item 2). Pinned against scipy's softmax/logsumexp on a
dense gather, page-permutation invariance, closed forms and the fold's
algebra."""
import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
import workloads
from helpers import dense_dequant, oracle_layer

W = workloads.small("att_small", seq_lens=(37, 130, 1), num_pages=16, block_size=16, q_heads=8, kv_heads=2,
                    head_dim=64)


def _full(w):
    return np.zeros(w.n_seq, np.int32), np.array(w.seq_lens, np.int32)


def test_matches_dense_softmax():
    x, cache = oracle_layer(W)
    out, lse2 = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads,
                                       W.head_dim, W.block_size)
    q = oracle.bf16_to_f64(x["q"])
    g = W.q_heads // W.kv_heads
    for s, L in enumerate(W.seq_lens):
        K, V = dense_dequant(cache, x["page_table"], s, L, W.block_size)
        for h in range(W.q_heads):
            sc = K[:, h // g, :] @ q[s, h] / np.sqrt(W.head_dim)
            p = softmax(sc)
            assert np.allclose(out[s, h], p @ V[:, h // g, :], rtol=1e-12, atol=1e-12)
            assert abs(lse2[s, h] - logsumexp(sc) / np.log(2)) < 1e-12


def test_page_permutation_invariance():
    x, cache = oracle_layer(W)
    ref = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads, W.head_dim,
                                 W.block_size)
    rng = np.random.default_rng(5)
    perm = rng.permutation(W.num_pages)          # new physical page of old page i
    moved = tuple(np.empty_like(a) for a in cache)
    for a, b in zip(cache, moved):
        b[perm] = a
    pt = np.where(x["page_table"] >= 0, perm[np.maximum(x["page_table"], 0)], -1).astype(np.int32)
    got = oracle.paged_attention(x["q"], moved, pt, *_full(W), W.q_heads, W.kv_heads, W.head_dim, W.block_size)
    assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1])


def test_single_token_context():
    x, cache = oracle_layer(W)
    out, lse2 = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads,
                                       W.head_dim, W.block_size)
    K, V = dense_dequant(cache, x["page_table"], 2, 1, W.block_size)   # sequence 2 has one token
    q = oracle.bf16_to_f64(x["q"])
    for h in range(W.q_heads):
        assert np.array_equal(out[2, h], V[0, h // 4])
        assert abs(lse2[2, h] - (K[0, h // 4] @ q[2, h]) / 8 / np.log(2)) < 1e-12


def test_identical_keys_give_mean_value():
    w = workloads.small("same_k", seq_lens=(50,), num_pages=4, block_size=16, q_heads=4, kv_heads=1, head_dim=64)
    x = workloads.host_layer(w)
    x["k_cache"][:] = x["k_cache"][0]
    x["k_new"][:] = x["k_cache"][0]
    x, cache = oracle_layer(w, inputs=x)
    out, lse2 = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(w), 4, 1, 64, 16)
    K, V = dense_dequant(cache, x["page_table"], 0, 50, 16)
    q = oracle.bf16_to_f64(x["q"])
    for h in range(4):
        assert np.allclose(out[0, h], V[:, 0].mean(0), atol=1e-13)
        assert abs(lse2[0, h] - ((K[0, 0] @ q[0, h]) / 8 / np.log(2) + np.log2(50))) < 1e-12


@pytest.mark.parametrize("n_split", [1, 2, 3, 7, 200])
def test_splits_fold_to_full_range(n_split):
    """Attention over token sub-ranges folded by log2-sum-exp equals the
    full-range attention, for any split count (empty splits included)."""
    x, cache = oracle_layer(W)
    full = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads, W.head_dim,
                                  W.block_size)
    L = np.array(W.seq_lens)
    o_parts, l_parts = [], []
    for i in range(n_split):
        tb = (L * i // n_split).astype(np.int32)
        te = (L * (i + 1) // n_split).astype(np.int32)
        o, l = oracle.paged_attention(x["q"], cache, x["page_table"], tb, te, W.q_heads, W.kv_heads, W.head_dim,
                                      W.block_size)
        o_parts.append(o.reshape(-1, W.head_dim))
        l_parts.append(l.reshape(-1))
    out, lse2 = oracle.lse_merge(np.stack(o_parts), np.stack(l_parts))
    assert np.allclose(out, full[0].reshape(-1, W.head_dim), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse2, full[1].reshape(-1), rtol=0, atol=1e-11)


def test_merge_identities():
    rng = np.random.default_rng(6)
    o = rng.standard_normal((1, 5, 16))
    l = rng.standard_normal((1, 5)) * 10
    out, lse2 = oracle.lse_merge(o, l)
    assert np.array_equal(out, o[0]) and np.array_equal(lse2, l[0])
    n = 6
    out, lse2 = oracle.lse_merge(np.repeat(o, n, 0), np.repeat(l, n, 0))
    assert np.allclose(out, o[0], atol=1e-14) and np.allclose(lse2, l[0] + np.log2(n), atol=1e-13)
    # parts with -inf carry no weight; all -inf gives 0 and -inf
    l2 = np.concatenate([l, np.full((1, 5), -np.inf)])
    o2 = np.concatenate([o, np.full((1, 5, 16), np.nan)])
    out, lse2 = oracle.lse_merge(o2, l2)
    assert np.array_equal(out, o[0]) and np.array_equal(lse2, l[0])
    out, lse2 = oracle.lse_merge(o2[1:], l2[1:])
    assert np.all(out == 0) and np.all(lse2 == -np.inf)
    # two parts: weights are 2^lse2 (a closed form)
    o3 = rng.standard_normal((2, 1, 4))
    l3 = np.array([[3.0], [1.0]])
    out, lse2 = oracle.lse_merge(o3, l3)
    assert np.allclose(out[0], (8 * o3[0, 0] + 2 * o3[1, 0]) / 10, atol=1e-15)
    assert abs(lse2[0] - np.log2(10)) < 1e-15


def test_softmax_scale_argument():
    x, cache = oracle_layer(W)
    a = oracle.paged_attention(x["q"], cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads, W.head_dim,
                               W.block_size)
    q2 = workloads.f32_to_bf16_bits(workloads.bf16_bits_to_f32(x["q"]) * 2)   # exact doubling
    b = oracle.paged_attention(q2, cache, x["page_table"], *_full(W), W.q_heads, W.kv_heads, W.head_dim,
                               W.block_size, softmax_scale=0.5 / np.sqrt(W.head_dim))
    assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-13)
