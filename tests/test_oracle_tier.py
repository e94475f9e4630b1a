"""Pins of the oracle's decode and prefill attention over a context held in
two pools (the host-placed tier: older tokens in a host pool, the rest in
the device pool), each against something other than itself.

On K/V that F4 stores exactly, the tiered result equals numpy's dense
attention over the concatenated input rows (host tokens first), for several
sequences with ragged device parts and empty tiers; moving whole pages
between the tiers (same tokens, same order) changes nothing; a host part
that is not whole pages is refused. Prefill: query i equals the dense
attention over the host part and the device tokens up to its own, and with
no host part the tiered prefill is the plain one."""
import numpy as np
import pytest

import oracle
import workloads
from test_oracle_prefill import _exact_rows

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _two_pools(rng, host_lens, dev_lens, block, hkv, d, v_group=32):
    """Exact-F4 rows of each sequence: the first host_lens[s] written to a
    permuted host pool, the rest to a permuted device pool."""
    def pool(lens, extra):
        n_pages = [-(-L // block) for L in lens]
        pages = sum(n_pages) + extra
        perm = rng.permutation(pages)
        pt = np.full((len(lens), max(n_pages + [1])), -1, np.int32)
        at = 0
        for s, n in enumerate(n_pages):
            pt[s, :n] = perm[at:at + n]
            at += n
        return oracle.empty_cache(pages, hkv, block, d, v_group=v_group), pt

    hc, hpt = pool(host_lens, 2)
    dc, dpt = pool(dev_lens, 1)
    ks, vs = [], []
    for s, (H, L) in enumerate(zip(host_lens, dev_lens)):
        k = _exact_rows(rng, H + L, hkv, d)
        v = _exact_rows(rng, H + L, hkv, d, v_group)
        for cache, pt, lo, n in ((hc, hpt, 0, H), (dc, dpt, H, L)):
            slots = np.array([pt[s, t // block] * block + t % block for t in range(n)], np.int64)
            assert oracle.kv_write_f4(k[lo:lo + n], v[lo:lo + n], slots, cache, hkv, d, block) == 0
        ks.append(k)
        vs.append(v)
    return hc, hpt, dc, dpt, ks, vs


@pytest.mark.parametrize("v_group", [32, 64])
def test_tiered_equals_dense_over_concatenation(v_group):
    rng = np.random.default_rng(11)
    block, hq, hkv, d = 16, 8, 2, 64
    host_lens, dev_lens = [48, 0, 32, 16], [5, 21, 0, 16]
    hc, hpt, dc, dpt, ks, vs = _two_pools(rng, host_lens, dev_lens, block, hkv, d, v_group)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((len(host_lens), hq, d)).astype(np.float32))
    out, lse2 = oracle.tiered_attention(q, hc, hpt, host_lens, dc, dpt, dev_lens, hq, hkv, d, block)
    for s in range(len(host_lens)):
        ob, lb = oracle.dense_attention(q[s], ks[s], vs[s])
        assert np.max(np.abs(out[s] - ob)) <= 1e-12
        assert np.max(np.abs(lse2[s] - lb)) <= 1e-12


def test_tiered_boundary_moves_change_nothing():
    rng = np.random.default_rng(12)
    block, hq, hkv, d = 16, 4, 1, 64
    total = 80
    k = _exact_rows(rng, total, hkv, d)
    v = _exact_rows(rng, total, hkv, d)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((1, hq, d)).astype(np.float32))
    results = []
    for host_pages in (0, 1, 3, 5):
        H = host_pages * block
        caches = []
        for lo, n in ((0, H), (H, total - H)):
            pages = max(1, -(-n // block))
            pt = rng.permutation(pages).astype(np.int32).reshape(1, -1)
            c = oracle.empty_cache(pages, hkv, block, d)
            slots = np.array([pt[0, t // block] * block + t % block for t in range(n)], np.int64)
            assert oracle.kv_write_f4(k[lo:lo + n], v[lo:lo + n], slots, c, hkv, d, block) == 0
            caches.append((c, pt))
        (hc, hpt), (dc, dpt) = caches
        results.append(oracle.tiered_attention(q, hc, hpt, [H], dc, dpt, [total - H], hq, hkv, d, block))
    for o, l in results[1:]:
        assert np.max(np.abs(o - results[0][0])) <= 1e-13
        assert np.max(np.abs(l - results[0][1])) <= 1e-13


def test_tiered_host_part_must_be_whole_pages():
    rng = np.random.default_rng(13)
    hc, hpt, dc, dpt, _, _ = _two_pools(rng, [32], [4], 16, 1, 64)
    q = np.zeros((1, 2, 64), np.uint16)
    with pytest.raises(ValueError):
        oracle.tiered_attention(q, hc, hpt, [20], dc, dpt, [4], 2, 1, 64, 16)


def test_tiered_prefill_equals_dense_on_each_prefix():
    """Query i of a chunk at device position p_i attends the whole host part
    and device tokens 0 .. p_i: dense attention over the first H + p_i + 1
    concatenated input rows."""
    rng = np.random.default_rng(14)
    block, hq, hkv, d = 16, 4, 2, 64
    H, L, n = 48, 37, 12                          # host tokens, device tokens, chunk at the device end
    hc, hpt, dc, dpt, ks, vs = _two_pools(rng, [H], [L], block, hkv, d)
    pos = np.arange(L - n, L)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((n, hq, d)).astype(np.float32))
    out, lse2 = oracle.tiered_prefill_attention(q, hc, hpt[0], H, dc, dpt[0], pos, hq, hkv, d, block)
    for i in range(n):
        t = H + int(pos[i]) + 1
        ob, lb = oracle.dense_attention(q[i], ks[0][:t], vs[0][:t])
        assert np.max(np.abs(out[i] - ob)) <= 1e-12
        assert np.max(np.abs(lse2[i] - lb)) <= 1e-12


def test_tiered_prefill_without_host_part_is_the_prefill():
    rng = np.random.default_rng(15)
    block, hq, hkv, d = 16, 4, 1, 64
    hc, hpt, dc, dpt, _, _ = _two_pools(rng, [0], [40], block, hkv, d)
    pos = np.arange(30, 40)
    q = workloads.f32_to_bf16_bits(rng.standard_normal((10, hq, d)).astype(np.float32))
    a = oracle.tiered_prefill_attention(q, hc, hpt[0], 0, dc, dpt[0], pos, hq, hkv, d, block)
    b = oracle.prefill_attention(q, dc, dpt[0], pos, hq, hkv, d, block)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
