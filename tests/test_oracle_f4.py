"""Pins of the oracle's F4 quantisation (mistral.rs PR "YaRN rope scaling,
4-bit F4 packed KV cache, ...", section 2: symmetric 4-bit values
(nibble - 8) * scale, 32 values per 16-byte cell) against a hand-derived cell,
a brute-force nearest-code search and closed-form error bounds."""
import numpy as np
import pytest

import oracle
import workloads
from conftest import read_golden


def _codes(b16):
    b = np.asarray(b16, dtype=np.uint8)
    return np.stack([b & 15, b >> 4], axis=-1).reshape(*b.shape[:-1], 32).astype(np.int64)


def _f32(x):
    return np.asarray(x, dtype=np.float32)


def test_hand_derived_cell():
    g, _ = read_golden("f4_cell_example.txt")
    x = workloads.f32_to_bf16_bits(_f32([(i % 15) - 7 for i in range(32)]))
    b, s = oracle.quantize_cell(x)
    assert s == int(g["scale"][0], 16)
    assert bytes(b).hex() == "".join(g["bytes"])


def test_zero_cell():
    b, s = oracle.quantize_cell(np.zeros(32, np.uint16))
    assert s == 0 and np.all(b == 0x88)


def _random_cells(n, seed, spread=3.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, 32)) * 10.0 ** rng.uniform(-spread, spread, (n, 1))
    return workloads.f32_to_bf16_bits(x.astype(np.float32))


def test_nearest_code_brute_force():
    """Each code is the grid point (c - 8) * scale nearest to x, ties to the
    even grid index, clamped to the 16 codes: found here by exhaustive search."""
    cells = _random_cells(3000, 0)
    # add exact half-way values: x = (k + 1/2) * scale for a scale of 1.0
    half = workloads.f32_to_bf16_bits(_f32([[7.0] + [((i % 14) - 7) + 0.5 for i in range(31)]]))
    cells = np.concatenate([cells, half])
    for x in cells:
        b, s = oracle.quantize_cell(x)
        sc = oracle.f16_to_f64(np.array([s]))[0]
        xv = oracle.bf16_to_f64(x)
        grid = (np.arange(16) - 8) * sc
        dist = np.abs(xv[:, None] - grid[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # ties: prefer the even signed value (c - 8 even <=> c even)
        want = np.where(cand.sum(1) > 1, np.argmax(cand & (np.arange(16) % 2 == 0), axis=1), np.argmax(cand, axis=1))
        assert np.array_equal(_codes(b), want)


def test_scale_and_error_bounds():
    cells = _random_cells(5000, 1)
    for x in cells:
        b, s = oracle.quantize_cell(x)
        sc = oracle.f16_to_f64(np.array([s]))[0]
        xv = oracle.bf16_to_f64(x)
        amax = np.max(np.abs(xv))
        # scale is amax/7 rounded once to fp16
        assert abs(sc - amax / 7) <= 0.5 * np.spacing(np.float16(sc)).astype(np.float64) * 1.0000001
        c = _codes(b)
        xhat = (c - 8) * sc
        if sc >= 2.0 ** -14:
            assert np.all(np.abs(xv - xhat) <= sc / 2 + 1e-300)
            assert not np.any(c == 0)  # -8 is never needed when scale ~ amax/7
            i = np.argmax(np.abs(xv))
            assert c[i] in (1, 15)


def test_dequant_requant_roundtrip():
    """Any code pattern reaching +-7 with an exactly representable product
    quantises back to itself."""
    rng = np.random.default_rng(2)
    for _ in range(500):
        c = rng.integers(1, 16, 32)
        c[rng.integers(0, 32)] = rng.choice([1, 15])
        scale = np.float16(rng.integers(1, 32) * 2.0 ** rng.integers(-10, 6)).astype(np.float64)
        x = workloads.f32_to_bf16_bits(_f32((c - 8) * scale))
        b, s = oracle.quantize_cell(x)
        assert oracle.f16_to_f64(np.array([s]))[0] == scale
        assert np.array_equal(_codes(b), c)


def test_saturating_scale():
    x = workloads.f32_to_bf16_bits(_f32([1e30] + [1.0] * 31))
    b, s = oracle.quantize_cell(x)
    assert s == 0x7BFF
    assert _codes(b)[0] == 15 and np.all(_codes(b)[1:] == 8)


@pytest.mark.parametrize("amax_bits", [0x3F80, 0x0080, 0x7F7F, 0x3380])
def test_every_bf16_value_maps_to_nearest(amax_bits):
    """Exhaustive over all finite bf16 values as the second element of a cell
    whose first element fixes amax (values above amax saturate the clamp)."""
    allb = np.arange(65536, dtype=np.uint16)
    fin = (allb & 0x7F80) != 0x7F80
    vals = allb[fin]
    cells = np.full((vals.size, 32), 0, np.uint16)
    cells[:, 0] = amax_bits
    cells[:, 1] = vals
    ka = np.empty((vals.size, 1, 256), np.uint16)
    ka[:, 0, :32] = cells
    ka[:, 0, 32:] = 0
    cache = oracle.empty_cache(vals.size, 1, 1, 256)
    bad = oracle.kv_write_f4(ka, ka, np.arange(vals.size), cache, 1, 256, 1)
    assert bad == 0
    kd, ks, _, _ = cache
    codes = _codes(kd[:, 0, 0, :16])
    sc = oracle.f16_to_f64(ks[:, 0, 0, 0])
    xv = oracle.bf16_to_f64(vals)
    am = np.maximum(np.abs(xv), oracle.bf16_to_f64(np.array([amax_bits]))[0])
    ok = sc > 0
    xhat = (codes[:, 1] - 8) * sc
    grid_err = np.abs(xv - xhat)
    # nearest-of-16 check, vectorised
    grid = (np.arange(16)[None, :] - 8) * sc[:, None]
    best = np.min(np.abs(xv[:, None] - grid), axis=1)
    assert np.all(grid_err[ok] == best[ok])
    assert np.all(codes[~ok] == 8)


def test_kv_write_layout_and_skips():
    """Slots land at page * B + offset; negative slots are skipped, slots past
    the pool are skipped and counted."""
    rng = np.random.default_rng(3)
    kv, d, B, P = 2, 64, 4, 5
    k = workloads.f32_to_bf16_bits(rng.standard_normal((4, kv, d)).astype(np.float32))
    v = workloads.f32_to_bf16_bits(rng.standard_normal((4, kv, d)).astype(np.float32))
    cache = oracle.empty_cache(P, kv, B, d)
    bad = oracle.kv_write_f4(k, v, np.array([7, -1, P * B, 0]), cache, kv, d, B)
    assert bad == 1
    kd, ks, vd, vs = cache
    for t, slot in [(0, 7), (3, 0)]:
        pg, off = divmod(slot, B)
        for h in range(kv):
            for c in range(d // 32):
                b, s = oracle.quantize_cell(k[t, h, 32 * c:32 * c + 32])
                assert np.array_equal(kd[pg, h, off, 16 * c:16 * c + 16], b) and ks[pg, h, off, c] == s
                b, s = oracle.quantize_cell(v[t, h, 32 * c:32 * c + 32])
                assert np.array_equal(vd[pg, h, off, 16 * c:16 * c + 16], b) and vs[pg, h, off, c] == s
    written = np.zeros((P, kv, B), bool)
    written[1, :, 3] = written[0, :, 0] = True
    assert np.all(kd[~written] == 0) and np.all(ks[~written] == 0)
    assert np.all(vd[~written] == 0) and np.all(vs[~written] == 0)


# --------------------------------------------------------------------------
# One V scale per token (the PR's own V layout: "one scale per token per V
# head"): the same quantiser over a group of head_dim values.

def _group_codes(b):
    b = np.asarray(b, dtype=np.uint8)
    return np.stack([b & 15, b >> 4], axis=-1).reshape(-1).astype(np.int64)


@pytest.mark.parametrize("n", [64, 128, 256])
def test_group_nearest_code_and_bound(n):
    """Per-token groups: every code is the nearest grid point (ties to even,
    clamped), |x - x_hat| <= scale / 2, and the largest element lands on code
    1 or 15 -- found by exhaustive search over the 16 codes."""
    rng = np.random.default_rng(n)
    for trial in range(200):
        x = workloads.f32_to_bf16_bits((rng.standard_normal(n) * 10.0 ** rng.uniform(-3, 3)).astype(np.float32))
        b, s = oracle.quantize_group(x)
        sc = oracle.f16_to_f64(np.array([s]))[0]
        xv = oracle.bf16_to_f64(x)
        assert s == int(oracle.f64_to_f16(np.array([np.abs(xv).max() / 7.0]))[0])
        grid = (np.arange(16) - 8) * sc
        dist = np.abs(xv[:, None] - grid[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        want = np.where(cand.sum(1) > 1, np.argmax(cand & (np.arange(16) % 2 == 0), axis=1), np.argmax(cand, axis=1))
        codes = _group_codes(b)
        assert np.array_equal(codes, want)
        assert np.all(np.abs(xv - (codes - 8) * sc) <= sc / 2 * (1 + 1e-12))
        assert codes[np.argmax(np.abs(xv))] in (1, 15)


def test_group_of_32_is_the_cell():
    for x in _random_cells(200, 4):
        assert oracle.quantize_group(x)[1] == oracle.quantize_cell(x)[1]
        assert np.array_equal(oracle.quantize_group(x)[0], oracle.quantize_cell(x)[0])


def test_group_zero_and_roundtrip():
    b, s = oracle.quantize_group(np.zeros(256, np.uint16))
    assert s == 0 and np.all(b == 0x88)
    rng = np.random.default_rng(8)
    codes = rng.integers(1, 16, 256)
    codes[17] = 15
    x = workloads.f32_to_bf16_bits(((codes - 8) * 0.125).astype(np.float32))
    b, s = oracle.quantize_group(x)
    assert oracle.f16_to_f64(np.array([s]))[0] == 0.125
    assert np.array_equal(_group_codes(b), codes)


def test_kv_write_per_token_v_scale():
    """kv_write_f4 into a cache with one V scale per token stores, for every
    (token, head), the group quantisation of the V row and the cell
    quantisation of the K row."""
    rng = np.random.default_rng(3)
    n, hkv, d, block = 20, 2, 256, 16
    k = workloads.f32_to_bf16_bits(rng.standard_normal((n, hkv, d)).astype(np.float32))
    v = workloads.f32_to_bf16_bits((rng.standard_normal((n, hkv, d)) * 3).astype(np.float32))
    cache = oracle.empty_cache(2, hkv, block, d, v_group=d)
    assert cache[3].shape == (2, hkv, block, 1)
    slots = rng.permutation(2 * block)[:n].astype(np.int64)
    assert oracle.kv_write_f4(k, v, slots, cache, hkv, d, block) == 0
    for t in range(n):
        page, off = divmod(int(slots[t]), block)
        for h in range(hkv):
            vb, vs = oracle.quantize_group(v[t, h])
            assert np.array_equal(cache[2][page, h, off], vb) and cache[3][page, h, off, 0] == vs
            for c in range(d // 32):
                kb, ks = oracle.quantize_cell(k[t, h, 32 * c:32 * c + 32])
                assert np.array_equal(cache[0][page, h, off, 16 * c:16 * c + 16], kb)
                assert cache[1][page, h, off, c] == ks
