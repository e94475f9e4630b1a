"""GPU parity of the split pass, the log2-sum-exp merge and the one-call
decode attention against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import ATOL_ATTN, attn_within, oracle_layer, split_bound, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _dev_cache(qkv, w, x, v_group=32):
    cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group)
    cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    cache.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    return cache


def _check_cache_equal(cache, ref):
    got = (to_host(cache.k_data), to_host(cache.k_scale).view(np.uint16), to_host(cache.v_data),
           to_host(cache.v_scale).view(np.uint16))
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def _run_attn(qkv, w, x, cache, num_splits=0, max_splits=0, softmax_scale=0.0):
    # a fixed split count needs that many workspace slots
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size,
                              max_splits=max_splits or num_splits)
    out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    att(out, to_dev(x["q"]), cache, to_dev(x["page_table"]), to_dev(x["seq_lens"]), lse2_out=lse,
        softmax_scale=softmax_scale, num_splits=num_splits, device_status=st)
    return to_host(out, np.uint16), to_host(lse), int(st.item())


def _oracle_attn(w, x, ref, softmax_scale=None):
    return oracle.paged_attention(x["q"], ref, x["page_table"], np.zeros(w.n_seq, np.int32), x["seq_lens"],
                                  w.q_heads, w.kv_heads, w.head_dim, w.block_size, softmax_scale)


def _assert_close(out, lse, ref_out, ref_lse):
    err, bound = attn_within(out, ref_out)
    assert np.all(err <= bound), f"max err {err.max():.3e} (excess {np.max(err - bound):.3e})"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.max(np.abs(lse[fin] - ref_lse[fin]), initial=0.0) <= 2e-4


CASES = [
    # seq_lens, block, q_heads, kv_heads, num_pages, num_splits
    ((4096,), 16, 16, 4, 256, 4),
    ((1,), 64, 16, 4, 4, 0),
    ((1, 2, 15, 16, 17), 16, 16, 4, 16, 3),
    ((63, 64, 65, 127, 129), 64, 8, 2, 16, 2),
    ((1000, 31, 4097), 32, 32, 4, 200, 0),
    ((333,), 64, 8, 8, 8, 1),
    ((2500,), 16, 4, 4, 300, 7),
    ((700, 1), 32, 16, 16, 30, 100),     # more splits than pages: empty splits
    ((5000, 3000, 10), 64, 16, 4, 140, 0),
    ((1000, 31, 4097, 0, 1), 32, 32, 4, 200, 0),  # an empty context and a single token among others
]


@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-B{c[1]}-G{c[2] // c[3]}-S{c[5]}" for c in CASES])
def test_decode_attention_matches_oracle(qkv, case):
    seq_lens, block, hq, hkv, pages, splits = case
    w = workloads.small("case", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous", head_scale=True)
    x, ref = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    _check_cache_equal(cache, ref)
    out, lse, st = _run_attn(qkv, w, x, cache, num_splits=splits)
    assert st == 0
    ref_out, ref_lse = _oracle_attn(w, x, ref)
    _assert_close(out, lse, ref_out, ref_lse)


# One V scale per token and head (the PR's own V layout): a subset of the
# cases above with every block size, ragged tails, empty contexts and splits.
VTOK_CASES = [CASES[i] for i in (0, 2, 3, 4, 6, 7, 9)]


@pytest.mark.parametrize("case", VTOK_CASES, ids=[f"L{c[0]}-B{c[1]}-G{c[2] // c[3]}-S{c[5]}" for c in VTOK_CASES])
def test_decode_attention_per_token_v_scale(qkv, case):
    seq_lens, block, hq, hkv, pages, splits = case
    w = workloads.small("vtok", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous", head_scale=True)
    x, ref = oracle_layer(w, v_group=w.head_dim)
    cache = _dev_cache(qkv, w, x, v_group=w.head_dim)
    assert cache.v_group == w.head_dim and cache.v_scale.shape[-1] == 1
    _check_cache_equal(cache, ref)
    out, lse, st = _run_attn(qkv, w, x, cache, num_splits=splits)
    assert st == 0
    ref_out, ref_lse = _oracle_attn(w, x, ref)
    _assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("v_group", [32, 256])
@pytest.mark.parametrize("num_splits", [1, 4, 9])
def test_split_partials_match_oracle_ranges(qkv, num_splits, v_group):
    """Each split's fp32 partial (o, lse2) equals exact attention over that
    split's page range; the fp32 partials meet 2e-3 with no bf16 allowance."""
    w = workloads.small("parts", seq_lens=(900, 130), num_pages=80, block_size=16, head_scale=True)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    rows = w.n_seq * w.q_heads
    o_parts = torch.empty((num_splits, rows, 256), dtype=torch.float32, device="cuda")
    l_parts = torch.empty((num_splits, rows), dtype=torch.float32, device="cuda")
    qkv.qkv_paged_decode_split_f4(o_parts, l_parts, to_dev(x["q"]), cache.k_data, cache.k_scale, cache.v_data,
                                  cache.v_scale, to_dev(x["page_table"]), to_dev(x["seq_lens"]), w.kv_heads,
                                  num_splits=num_splits)
    o_parts, l_parts = to_host(o_parts), to_host(l_parts)
    for i in range(num_splits):
        tb, te = [], []
        for L in w.seq_lens:
            n = -(-L // w.block_size)
            tb.append(split_bound(i, n, num_splits, w.block_size, 256) * w.block_size)
            te.append(min(split_bound(i + 1, n, num_splits, w.block_size, 256) * w.block_size, L))
        ro, rl = oracle.paged_attention(x["q"], ref, x["page_table"], tb, te, w.q_heads, w.kv_heads, 256,
                                        w.block_size)
        ro, rl = ro.reshape(rows, 256), rl.reshape(rows)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l_parts[i]), fin)
        assert np.max(np.abs(o_parts[i][fin] - ro[fin]), initial=0.0) <= ATOL_ATTN
        assert np.max(np.abs(l_parts[i][fin] - rl[fin]), initial=0.0) <= 2e-4


# part counts: 1, 5 and 8 (the one-warp-per-row merge for up to 8 parts:
# the prefill's context split, short decode plans), the automatic plan's 37
# on a B200, the 1M-token workload's 148 (>= 128 weighted parts per row),
# and 600, past the merge's first rounds of 256 parts (8 warps x 32 lanes)
# into its third
@pytest.mark.parametrize("n", [1, 5, 8, 37, 148, 600])
def test_lse_merge_matches_oracle(qkv, n):
    rng = np.random.default_rng(21 + n)
    rows, d = 48, 256
    o = rng.standard_normal((n, rows, d)).astype(np.float32)
    l = (rng.standard_normal((n, rows)) * 30).astype(np.float32)
    l[rng.random((n, rows)) < 0.2] = -np.inf
    l[:, 5] = -np.inf                     # a row without any weighted part
    if n > 512:
        l[:512, 7] = -np.inf              # weighted parts only in the last round (past part 512)
        l[600 - 3, 9] = 400.0             # the row's maximum in the last round
    o[np.isinf(l)] = np.nan               # unweighted parts are never read
    out = torch.empty((rows, d), dtype=torch.int16, device="cuda")
    lo = torch.empty(rows, dtype=torch.float32, device="cuda")
    qkv.qkv_lse_merge(to_dev(o), to_dev(l), out, lo)
    ref_o, ref_l = oracle.lse_merge(o.astype(np.float64), l.astype(np.float64))
    got = workloads.bf16_bits_to_f32(to_host(out, np.uint16)).astype(np.float64)
    from helpers import bf16_ulp
    assert np.all(np.abs(got - ref_o) <= 1e-5 + 0.5 * bf16_ulp(ref_o) * 1.0001)
    lo = to_host(lo)
    assert np.array_equal(np.isfinite(lo), np.isfinite(ref_l))
    fin = np.isfinite(ref_l)
    assert np.max(np.abs(lo[fin] - ref_l[fin])) <= 1e-5 * np.max(np.abs(ref_l[fin]))
    assert np.all(got[5] == 0)
    # rows with at least 128 weighted parts are covered at n >= 148
    assert np.max(np.isfinite(l).sum(0)) >= min(n, 128) * 0.7


def test_split_count_above_workspace_refused(qkv):
    """A fixed split count larger than the workspace's split slots is an
    argument error, never silently reduced."""
    w = workloads.small("toomany", seq_lens=(640,), num_pages=10, block_size=64)
    x, _ = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size, max_splits=4)
    out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
    with pytest.raises(qkv.QkvError) as e:
        att(out, to_dev(x["q"]), cache, to_dev(x["page_table"]), to_dev(x["seq_lens"]), num_splits=5)
    assert e.value.code == 1


@pytest.mark.parametrize("v_group", [32, 256])
def test_148_splits_all_weighted(qkv, v_group):
    """The 1M-token workload's plan shape at a size the oracle finishes: 148
    splits of every sequence, each holding pages (so every query row merges
    148 weighted parts), checked part by part and after the merge."""
    S = 148
    w = workloads.small("s148", seq_lens=(S * 2 * 64 - 17, S * 64 + 5), num_pages=S * 3 + 1, block_size=64,
                        head_scale=True, page_alloc="interleaved", k_outlier_frac=0.01)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size, max_splits=S)
    out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    att(out, to_dev(x["q"]), cache, to_dev(x["page_table"]), to_dev(x["seq_lens"]), lse2_out=lse, num_splits=S,
        device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _, l_parts = att.partials(w.n_seq, w.q_heads, w.head_dim)
    assert np.all(np.isfinite(to_host(l_parts)).sum(0) == S)
    ref_out, ref_lse = _oracle_attn(w, x, ref)
    _assert_close(to_host(out, np.uint16), to_host(lse), ref_out, ref_lse)


def test_page_permutation_invariance_gpu(qkv):
    w = workloads.small("perm", seq_lens=(1500,), num_pages=30, block_size=64)
    x, ref = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    out1, lse1, _ = _run_attn(qkv, w, x, cache, num_splits=5)
    perm = np.random.default_rng(3).permutation(w.num_pages)
    for t in (cache.k_data, cache.k_scale, cache.v_data, cache.v_scale):
        t[torch.from_numpy(perm).cuda()] = t.clone()
    x2 = dict(x)
    x2["page_table"] = np.where(x["page_table"] >= 0, perm[np.maximum(x["page_table"], 0)], -1).astype(np.int32)
    out2, lse2, _ = _run_attn(qkv, w, x2, cache, num_splits=5)
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


@pytest.mark.parametrize("v_group", [32, 256])
def test_single_token_is_exact_value(qkv, v_group):
    w = workloads.small("one", seq_lens=(1, 1), num_pages=2, block_size=64)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    out, lse, st = _run_attn(qkv, w, x, cache)
    ro, rl = _oracle_attn(w, x, ref)
    # p = 1 exactly: the output is the dequantised value, rounded to bf16 once
    assert np.array_equal(out, oracle.f64_to_bf16(ro))


def test_empty_and_bad_inputs_flag(qkv):
    w = workloads.small("edge", seq_lens=(100, 64), num_pages=4, block_size=64)
    x, ref = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    x2 = dict(x)
    x2["seq_lens"] = np.array([0, 64], np.int32)       # an empty context
    out, lse, st = _run_attn(qkv, w, x2, cache, num_splits=2)
    assert st == 0
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    x3 = dict(x)
    pt = x["page_table"].copy()
    pt[1, 0] = 999                                     # page id outside the pool
    x3["page_table"] = pt
    out, lse, st = _run_attn(qkv, w, x3, cache, num_splits=1)
    assert st & qkv.DEV_BAD_PAGE
    x4 = dict(x)
    x4["seq_lens"] = np.array([100, 10 ** 6], np.int32)  # longer than its page-table row
    out, lse, st = _run_attn(qkv, w, x4, cache, num_splits=1)
    assert st & qkv.DEV_BAD_SEQLEN


def test_softmax_scale_argument_gpu(qkv):
    w = workloads.small("scale", seq_lens=(777,), num_pages=16, block_size=64)
    x, ref = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    out, lse, st = _run_attn(qkv, w, x, cache, softmax_scale=0.3)
    ro, rl = _oracle_attn(w, x, ref, softmax_scale=0.3)
    _assert_close(out, lse, ro, rl)


# head_dim 128: 64-byte rows (64-byte TMA swizzle), two cell pairs in Q K^T,
# one cell per warp in P V; every block size, G 1/2/4/8, ragged and empty
# contexts, both V layouts
D128_CASES = [
    # seq_lens, block, q_heads, kv_heads, num_pages, num_splits
    ((4096,), 16, 16, 4, 256, 4),
    ((1, 2, 15, 16, 17), 16, 16, 4, 16, 3),
    ((63, 64, 65, 127, 129), 64, 8, 2, 16, 2),
    ((1000, 31, 4097, 0, 1), 32, 32, 4, 200, 0),
    ((333,), 64, 8, 8, 8, 1),
    ((5000, 3000, 10), 64, 16, 4, 140, 0),
]


@pytest.mark.parametrize("v_group", [32, 128])
@pytest.mark.parametrize("case", D128_CASES, ids=[f"L{c[0]}-B{c[1]}-G{c[2] // c[3]}-S{c[5]}" for c in D128_CASES])
def test_decode_attention_head_dim_128(qkv, case, v_group):
    seq_lens, block, hq, hkv, pages, splits = case
    w = workloads.small("d128", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        head_dim=128, page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous",
                        head_scale=True)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    _check_cache_equal(cache, ref)
    out, lse, st = _run_attn(qkv, w, x, cache, num_splits=splits)
    assert st == 0
    ref_out, ref_lse = _oracle_attn(w, x, ref)
    _assert_close(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("v_group", [32, 128])
def test_split_partials_head_dim_128(qkv, v_group):
    """Per-split fp32 partials at head_dim 128 against the oracle's sub-range
    attention (strict 2e-3, no bf16 allowance)."""
    S = 9   # >= 8: the plan's shorter first splits
    w = workloads.small("parts128", seq_lens=(1900, 130), num_pages=140, block_size=16, head_dim=128, head_scale=True)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    rows = w.n_seq * w.q_heads
    o_parts = torch.empty((S, rows, 128), dtype=torch.float32, device="cuda")
    l_parts = torch.empty((S, rows), dtype=torch.float32, device="cuda")
    qkv.qkv_paged_decode_split_f4(o_parts, l_parts, to_dev(x["q"]), cache.k_data, cache.k_scale, cache.v_data,
                                  cache.v_scale, to_dev(x["page_table"]), to_dev(x["seq_lens"]), w.kv_heads,
                                  num_splits=S)
    o_parts, l_parts = to_host(o_parts), to_host(l_parts)
    for i in range(S):
        tb, te = [], []
        for L in w.seq_lens:
            n = -(-L // w.block_size)
            tb.append(split_bound(i, n, S, w.block_size, 128) * w.block_size)
            te.append(min(split_bound(i + 1, n, S, w.block_size, 128) * w.block_size, L))
        ro, rl = oracle.paged_attention(x["q"], ref, x["page_table"], tb, te, w.q_heads, w.kv_heads, 128,
                                        w.block_size)
        ro, rl = ro.reshape(rows, 128), rl.reshape(rows)
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l_parts[i]), fin)
        assert np.max(np.abs(o_parts[i][fin] - ro[fin]), initial=0.0) <= ATOL_ATTN
        assert np.max(np.abs(l_parts[i][fin] - rl[fin]), initial=0.0) <= 2e-4


@pytest.mark.parametrize("v_group", [32, 128])
def test_single_token_is_exact_value_head_dim_128(qkv, v_group):
    w = workloads.small("one128", seq_lens=(1, 1), num_pages=2, block_size=64, head_dim=128)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = _dev_cache(qkv, w, x, v_group=v_group)
    out, lse, st = _run_attn(qkv, w, x, cache)
    ro, rl = _oracle_attn(w, x, ref)
    assert np.array_equal(out, oracle.f64_to_bf16(ro))


def test_unsupported_shapes_raise(qkv):
    """head_dim 256 and 128 are the compiled decode shapes; 192 is refused."""
    w = workloads.small("bad", seq_lens=(10,), num_pages=2, block_size=64, head_dim=192)
    x, _ = oracle_layer(w)
    cache = _dev_cache(qkv, w, x)
    with pytest.raises(qkv.QkvError) as e:
        _run_attn(qkv, w, x, cache)
    assert e.value.code == 2


def test_workspace_reuse_across_calls(qkv):
    """One workspace serves calls with different inputs, split counts and
    sequence counts in a row; each matches the oracle."""
    att = qkv.DecodeAttention(3, 16, 4, 256, 64, max_splits=16)
    calls = [
        (workloads.small("reuse_a", seq_lens=(3000, 70, 1), num_pages=60, block_size=64, head_scale=True,
                         page_alloc="interleaved"), 0),
        (workloads.small("reuse_b", seq_lens=(1200, 4000), num_pages=90, block_size=64, seed=5,
                         page_alloc="interleaved"), 7),
        (workloads.small("reuse_c", seq_lens=(64,), num_pages=2, block_size=64, seed=9), 16),
    ]
    for w, splits in calls:
        x, ref = oracle_layer(w)
        cache = _dev_cache(qkv, w, x)
        out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
        lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        att(out, to_dev(x["q"]), cache, to_dev(x["page_table"]), to_dev(x["seq_lens"]), lse2_out=lse,
            num_splits=splits, device_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ref_out, ref_lse = _oracle_attn(w, x, ref)
        _assert_close(to_host(out, np.uint16), to_host(lse), ref_out, ref_lse)
