"""The dense bf16 attention of the oracle (the reference the F4 cache is
measured against) and the F4-vs-bf16 deviation report.

Pins: on K/V that F4 stores exactly (each cell a power-of-two scale times
codes -7..7, one element at +-7) the dense attention over the bf16 values and
the paged attention over the F4 cache agree to rounding; every score of the
F4 cache lies within the bound that the per-element error |x - x_hat| <=
scale / 2 implies; the report runs."""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _exact_rows(rng, n, hkv, d):
    """bf16 bits of rows whose every 32-value cell is s * (c - 8), s = 2^-e,
    with codes c in 1..15 and one element at +-7 s (so amax / 7 = s)."""
    codes = rng.integers(1, 16, size=(n, hkv, d // 32, 32))
    codes[..., 0] = rng.choice([1, 15], size=(n, hkv, d // 32))
    e = rng.integers(0, 6, size=(n, hkv, d // 32, 1))
    x = (codes - 8) * np.ldexp(1.0, -e)
    return workloads.f32_to_bf16_bits(x.reshape(n, hkv, d).astype(np.float32)), codes


def test_dense_equals_paged_on_exact_f4_values():
    rng = np.random.default_rng(11)
    hq, hkv, d, block, T = 8, 2, 256, 16, 100
    k, kc = _exact_rows(rng, T, hkv, d)
    v, vc = _exact_rows(rng, T, hkv, d)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((1, hq, d)).astype(np.float32))
    pages = -(-T // block)
    cache = oracle.empty_cache(pages, hkv, block, d)
    perm = rng.permutation(pages)
    pt = perm[None, :].astype(np.int32)
    slots = np.array([perm[t // block] * block + t % block for t in range(T)], np.int64)
    assert oracle.kv_write_f4(k, v, slots, cache, hkv, d, block) == 0
    # the F4 codes are the ones built in (lossless)
    kd = cache[0][perm[0], 0, 0]
    assert np.array_equal(kd & 0xF, kc[0, 0].reshape(-1)[0::2]) and np.array_equal(kd >> 4, kc[0, 0].reshape(-1)[1::2])
    o4, l4 = oracle.paged_attention(q, cache, pt, [0], [T], hq, hkv, d, block)
    ob, lb = oracle.dense_attention(q[0], k, v)
    assert np.max(np.abs(o4[0] - ob)) <= 1e-12
    assert np.max(np.abs(l4[0] - lb)) <= 1e-12


def test_dense_attention_definition():
    """Against an independent evaluation: scipy's softmax and logsumexp."""
    from scipy.special import logsumexp, softmax
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 64))
    k = rng.standard_normal((37, 2, 64))
    v = rng.standard_normal((37, 2, 64))
    o, l = oracle.dense_attention(q, k, v, softmax_scale=0.2)
    for h in range(4):
        s = k[:, h // 2, :] @ q[h] * 0.2
        assert np.allclose(o[h], softmax(s) @ v[:, h // 2, :], rtol=0, atol=1e-13)
        assert abs(l[h] - logsumexp(s) / np.log(2)) <= 1e-13
    o0, l0 = oracle.dense_attention(q, k[:0], v[:0])
    assert np.all(o0 == 0) and np.all(np.isneginf(l0))


def test_f4_score_error_within_cell_bound():
    """|q.k_hat - q.k| <= sum over cells of (scale / 2) * sum |q| over the
    cell, for every token and head (from |x - x_hat| <= scale / 2)."""
    rng = np.random.default_rng(5)
    hkv, d, block, T = 2, 256, 16, 64
    k = workloads.f32_to_bf16_bits((rng.standard_normal((T, hkv, d)) * rng.uniform(0.1, 30, (T, hkv, 1)))
                                   .astype(np.float32))
    v = np.zeros_like(k)
    cache = oracle.empty_cache(T // block, hkv, block, d)
    slots = np.arange(T, dtype=np.int64)
    oracle.kv_write_f4(k, v, slots, cache, hkv, d, block)
    kd, ks = cache[0], cache[1]
    codes = np.stack([kd & 0xF, kd >> 4], axis=-1).reshape(T // block, hkv, block, d).astype(np.float64) - 8
    scale = oracle.f16_to_f64(ks)                                      # [pages][hkv][block][cells]
    khat = (codes.reshape(T // block, hkv, block, d // 32, 32) * scale[..., None]).reshape(T // block, hkv, block, d)
    khat = khat.transpose(0, 2, 1, 3).reshape(T, hkv, d)
    kf = oracle.bf16_to_f64(k)
    q = rng.standard_normal((hkv, d))
    err = np.abs(np.einsum("thd,hd->th", khat - kf, q))
    sc = scale.transpose(0, 2, 1, 3).reshape(T, hkv, d // 32)
    bound = np.einsum("thc,hc->th", sc / 2, np.abs(q).reshape(hkv, d // 32, 32).sum(-1))
    assert np.all(err <= bound * (1 + 1e-12) + 1e-300)
    assert err.max() > 0.05 * bound.max()   # not vacuous


def test_deviation_report_runs_small():
    from oracle import f4_deviation
    r = f4_deviation.deviation(f4_deviation.sample(workloads.TINY_4K, 1024))
    assert r["tokens"] == 1024
    assert 0 < r["rel_out"] < 0.5 and np.isfinite(r["max_abs_lse2"])


def test_dense_equals_paged_per_token_v_scale():
    """Per-token V scales: on V rows that one power-of-two scale per row
    stores exactly, paged attention over the F4 cache equals the dense bf16
    attention (K stored exactly per cell as before)."""
    rng = np.random.default_rng(12)
    hq, hkv, d, block, T = 8, 2, 256, 16, 90
    k, _ = _exact_rows(rng, T, hkv, d)
    vcodes = rng.integers(1, 16, size=(T, hkv, d))
    vcodes[..., 5] = 15
    vexp = rng.integers(0, 6, size=(T, hkv, 1))
    v = workloads.f32_to_bf16_bits(((vcodes - 8) * np.ldexp(1.0, -vexp)).astype(np.float32))
    q = workloads.f32_to_bf16_bits(rng.standard_normal((1, hq, d)).astype(np.float32))
    pages = -(-T // block)
    cache = oracle.empty_cache(pages, hkv, block, d, v_group=d)
    pt = np.arange(pages, dtype=np.int32)[None, :]
    assert oracle.kv_write_f4(k, v, np.arange(T, dtype=np.int64), cache, hkv, d, block) == 0
    o4, l4 = oracle.paged_attention(q, cache, pt, [0], [T], hq, hkv, d, block)
    ob, lb = oracle.dense_attention(q[0], k, v)
    assert np.max(np.abs(o4[0] - ob)) <= 1e-12 and np.max(np.abs(l4[0] - lb)) <= 1e-12
