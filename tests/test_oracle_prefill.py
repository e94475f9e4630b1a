"""Pins of the oracle's paged -> contiguous gather and of its chunked causal
prefill attention, each against something other than itself.

Gather: on K/V that F4 stores exactly (every scale group a power-of-two scale
times codes -7..7 with one element at +-7), writing and gathering back
returns the input bits; a permutation of the physical pages changes nothing;
tokens on a page id outside the pool come back as zero rows and are counted.

Prefill: query i of a chunk at position p_i equals the dense attention of
that query over the first p_i + 1 gathered rows (an independent route:
numpy's dense definition, itself pinned to scipy); the first token attends
itself alone, so its output is its dequantised value; and changing the cache
after p_i leaves query i unchanged (causality)."""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _exact_rows(rng, n, hkv, d, group=32):
    """bf16 bits of rows whose every `group`-value scale group is s * code,
    s = 2^-e, codes in -7..7 with one element at +-7 (so amax / 7 = s)."""
    codes = rng.integers(-7, 8, size=(n, hkv, d // group, group))
    codes[..., 0] = rng.choice([-7, 7], size=(n, hkv, d // group))
    e = rng.integers(0, 8, size=(n, hkv, d // group, 1))
    x = codes * np.ldexp(1.0, -e)
    return workloads.f32_to_bf16_bits(x.reshape(n, hkv, d).astype(np.float32))


def _pool(rng, seq_lens, block, hkv, d, v_group=32, extra_pages=3):
    """Exact-F4 K/V of several sequences in one interleaved, permuted pool."""
    n_pages = [-(-L // block) for L in seq_lens]
    pages = sum(n_pages) + extra_pages
    perm = rng.permutation(pages)
    pt = np.full((len(seq_lens), max(n_pages + [1])), -1, np.int32)
    at = 0
    for s, n in enumerate(n_pages):
        pt[s, :n] = perm[at:at + n]
        at += n
    cache = oracle.empty_cache(pages, hkv, block, d, v_group=v_group)
    ks, vs = [], []
    for s, L in enumerate(seq_lens):
        k = _exact_rows(rng, L, hkv, d)
        v = _exact_rows(rng, L, hkv, d, v_group)
        slots = np.array([pt[s, t // block] * block + t % block for t in range(L)], np.int64)
        assert oracle.kv_write_f4(k, v, slots, cache, hkv, d, block) == 0
        ks.append(k)
        vs.append(v)
    return cache, pt, ks, vs


@pytest.mark.parametrize("v_group", [32, 128])
def test_gather_returns_exact_f4_input(v_group):
    rng = np.random.default_rng(5)
    seq_lens, block, hkv, d = [37, 0, 64, 129], 16, 2, 128
    cache, pt, ks, vs = _pool(rng, seq_lens, block, hkv, d, v_group)
    start = np.concatenate([[0], np.cumsum(seq_lens)[:-1]]).astype(np.int64)
    ko, vo, bad = oracle.gather_kv_f4(cache, pt, seq_lens, start, hkv, d, block)
    assert bad == 0 and ko.shape == (sum(seq_lens), hkv, d)
    for s, L in enumerate(seq_lens):
        assert np.array_equal(ko[start[s]:start[s] + L], ks[s])
        assert np.array_equal(vo[start[s]:start[s] + L], vs[s])


def test_gather_page_permutation_and_bad_pages():
    rng = np.random.default_rng(6)
    block, hkv, d = 16, 2, 64
    cache, pt, ks, vs = _pool(rng, [50], block, hkv, d, extra_pages=0)
    ko, vo, _ = oracle.gather_kv_f4(cache, pt, [50], [0], hkv, d, block)
    perm = rng.permutation(cache[0].shape[0])
    moved = tuple(np.empty_like(a) for a in cache)
    for a, b in zip(cache, moved):
        b[perm] = a
    ko2, vo2, _ = oracle.gather_kv_f4(moved, perm[pt].astype(np.int32), [50], [0], hkv, d, block)
    assert np.array_equal(ko, ko2) and np.array_equal(vo, vo2)
    pt_bad = pt.copy()
    pt_bad[0, 1] = cache[0].shape[0]          # one page past the pool: 16 tokens
    ko3, vo3, bad = oracle.gather_kv_f4(cache, pt_bad, [50], [0], hkv, d, block)
    assert bad == 16
    assert np.all(ko3[16:32] == 0) and np.all(vo3[16:32] == 0)
    assert np.array_equal(ko3[:16], ko[:16]) and np.array_equal(ko3[32:], ko[32:])


def _chunk(rng, L, n, hq, hkv, d, block):
    cache, pt, ks, vs = _pool(rng, [L], block, hkv, d)
    pos = np.arange(L - n, L, dtype=np.int64)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((n, hq, d)).astype(np.float32))
    return cache, pt, ks[0], vs[0], pos, q


def test_prefill_equals_dense_on_each_prefix():
    rng = np.random.default_rng(7)
    L, n, hq, hkv, d, block = 90, 20, 4, 2, 64, 16
    cache, pt, k, v, pos, q = _chunk(rng, L, n, hq, hkv, d, block)
    out, lse2 = oracle.prefill_attention(q, cache, pt[0], pos, hq, hkv, d, block)
    assert out.shape == (n, hq, d) and lse2.shape == (n, hq)
    for i in range(n):
        p = int(pos[i])
        ob, lb = oracle.dense_attention(q[i], k[:p + 1], v[:p + 1])
        assert np.max(np.abs(out[i] - ob)) <= 1e-12
        assert np.max(np.abs(lse2[i] - lb)) <= 1e-12


def test_prefill_first_token_and_causality():
    rng = np.random.default_rng(8)
    L, hq, hkv, d, block = 40, 4, 2, 64, 16
    cache, pt, k, v, _, _ = _chunk(rng, L, 1, hq, hkv, d, block)
    pos = np.arange(0, L, dtype=np.int64)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((L, hq, d)).astype(np.float32))
    out, _ = oracle.prefill_attention(q, cache, pt[0], pos, hq, hkv, d, block)
    # position 0 attends itself alone: the output is its value exactly
    for h in range(hq):
        assert np.array_equal(out[0, h], oracle.bf16_to_f64(v[0, h // (hq // hkv)]))
    # rewriting tokens 25.. leaves queries 0..24 unchanged
    k2 = _exact_rows(rng, L - 25, hkv, d)
    slots = np.array([pt[0, t // block] * block + t % block for t in range(25, L)], np.int64)
    assert oracle.kv_write_f4(k2, k2, slots, cache, hkv, d, block) == 0
    out2, _ = oracle.prefill_attention(q, cache, pt[0], pos, hq, hkv, d, block)
    assert np.array_equal(out[:25], out2[:25])
    assert not np.array_equal(out[25:], out2[25:])
