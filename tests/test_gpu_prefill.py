"""GPU parity of the chunked causal prefill attention over the paged F4
cache (qkv_paged_prefill_attn_f4, tcgen05) with the oracle: every query of a
chunk against exact attention over its causal prefix, for ragged chunk sizes,
empty and long prefixes, every GQA ratio, three block sizes, both V scale
layouts and head_dim 256 and 128; bad page ids are flagged."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import attn_within, bf16_ulp, oracle_layer, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _setup(qkv, L, n_q, block, hq, hkv, v_group=256, pages=None, seed=0, head_scale=True, outliers=0.0,
           head_dim=256):
    w = workloads.small("prefill", seq_lens=(L,), num_pages=pages or -(-L // block) + 3, block_size=block,
                        q_heads=hq, kv_heads=hkv, head_scale=head_scale, seed=seed, k_outlier_frac=outliers,
                        head_dim=head_dim)
    x, ref = oracle_layer(w, v_group=v_group)
    cache = qkv.PagedF4Cache.allocate(w.num_pages, hkv, block, head_dim, v_group=v_group)
    cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    cache.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    q = workloads.chunk_queries_host(w, 0, n_q)
    return w, x, ref, cache, q


def _run(qkv, w, x, cache, q, prefix, page_table=None, softmax_scale=0.0, num_splits=1, ws_splits=0):
    n_q = q.shape[0]
    out = torch.full((n_q, w.q_heads, w.head_dim), 0x7FC1, dtype=torch.int16, device="cuda")
    lse = torch.empty((n_q, w.q_heads), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pt = x["page_table"][0] if page_table is None else page_table
    nb = qkv.qkv_paged_prefill_workspace_bytes(n_q, w.q_heads, w.head_dim, ws_splits) if ws_splits > 1 else 0
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    qkv.qkv_paged_prefill_attn_f4(out, to_dev(q), cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                                  to_dev(np.ascontiguousarray(pt)), prefix, w.kv_heads, lse2_out=lse,
                                  softmax_scale=softmax_scale, num_splits=num_splits, workspace=ws,
                                  device_status=st)
    return to_host(out, np.uint16), to_host(lse), int(st.item())


def _check(out, lse, ref_out, ref_lse):
    err, bound = attn_within(out, ref_out)
    assert np.all(err <= bound), f"max err {err.max():.3e} (excess {np.max(err - bound):.3e})"
    assert np.max(np.abs(lse - ref_lse)) <= 2e-3


CASES = [
    # L (context incl. the chunk), n_q, block, q_heads, kv_heads
    (100, 100, 16, 16, 4),      # no prefix: the whole sequence is the chunk, 4 ragged query blocks
    (700, 64, 64, 16, 4),       # prefix 636
    (1600, 257, 32, 16, 4),     # several stages, a ragged last query block
    (300, 129, 64, 4, 4),       # GQA 1: 128 queries per block
    (400, 130, 16, 8, 4),       # GQA 2
    (333, 40, 64, 16, 2),       # GQA 8
    (65, 1, 64, 16, 4),         # one query at the end of the context
]


@pytest.mark.parametrize("v_group", [32, 256])
@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-n{c[1]}-B{c[2]}-G{c[3] // c[4]}" for c in CASES])
def test_prefill_matches_oracle(qkv, case, v_group):
    L, n_q, block, hq, hkv = case
    w, x, ref, cache, q = _setup(qkv, L, n_q, block, hq, hkv, v_group)
    prefix = L - n_q
    out, lse, st = _run(qkv, w, x, cache, q, prefix)
    assert st == 0
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(prefix, L), hq, hkv, 256, block)
    _check(out, lse, ro, rl)


D128_CASES = [
    (100, 100, 16, 16, 4),
    (1600, 257, 32, 16, 4),
    (300, 129, 64, 4, 4),
    (400, 130, 16, 8, 4),
    (333, 40, 64, 16, 2),
    (65, 1, 64, 16, 4),
]


@pytest.mark.parametrize("v_group", [32, 128])
@pytest.mark.parametrize("case", D128_CASES, ids=[f"L{c[0]}-n{c[1]}-B{c[2]}-G{c[3] // c[4]}" for c in D128_CASES])
def test_prefill_d128_matches_oracle(qkv, case, v_group):
    """head_dim 128: 64-byte packed rows, one 64-dim chunk of V per CTA of the pair."""
    L, n_q, block, hq, hkv = case
    w, x, ref, cache, q = _setup(qkv, L, n_q, block, hq, hkv, v_group, head_dim=128)
    prefix = L - n_q
    out, lse, st = _run(qkv, w, x, cache, q, prefix)
    assert st == 0
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(prefix, L), hq, hkv, 128, block)
    _check(out, lse, ro, rl)


def test_prefill_d128_context_split_and_first_query(qkv):
    """head_dim 128 with the context in three parts, and query 0 of a chunk
    without prefix (token 0's value within one bf16 ulp)."""
    L, n_q = 1600, 257
    w, x, ref, cache, q = _setup(qkv, L, n_q, 32, 16, 4, 32, head_dim=128)
    out, lse, st = _run(qkv, w, x, cache, q, L - n_q, num_splits=3, ws_splits=3)
    assert st == 0
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(L - n_q, L), 16, 4, 128, 32)
    _check(out, lse, ro, rl)
    w, x, ref, cache, q = _setup(qkv, 70, 70, 16, 16, 4, head_dim=128, v_group=128)
    out, _, st = _run(qkv, w, x, cache, q, 0)
    ro, _ = oracle.prefill_attention(q[:1], ref, x["page_table"][0], np.arange(0, 1), 16, 4, 128, 16)
    got = oracle.bf16_to_f64(out[0])
    assert st == 0 and np.all(np.abs(got - ro[0]) <= bf16_ulp(ro[0]))


@pytest.mark.parametrize("splits", [(2, 2), (3, 3), (0, 8)], ids=["S2", "S3", "auto"])
def test_prefill_context_split(qkv, splits):
    """Each query block's context in parts, partials folded by the merge."""
    num_splits, ws_splits = splits
    L, n_q = 1600, 257
    w, x, ref, cache, q = _setup(qkv, L, n_q, 32, 16, 4, 32)
    out, lse, st = _run(qkv, w, x, cache, q, L - n_q, num_splits=num_splits, ws_splits=ws_splits)
    assert st == 0
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(L - n_q, L), 16, 4, 256, 32)
    _check(out, lse, ro, rl)


@pytest.mark.parametrize("case", [(700, 64, 64, 16, 4), (200, 64, 64, 16, 4)], ids=["L700-n64", "L200-n64"])
def test_prefill_repeated_calls_hold_the_last_stages(qkv, case):
    """One short-context chunk 16 times over: every output must hold the
    P.V products of the last two stages. (The epilogue once took O as done
    on a parity wait that the per-stage barrier could pass a phase early,
    when the last P.V finished late: lse right, the output without those
    stages, in about one call of a few hundred.)"""
    L, n_q, block, hq, hkv = case
    w, x, ref, cache, q = _setup(qkv, L, n_q, block, hq, hkv, 32)
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(L - n_q, L), hq, hkv, 256, block)
    for _ in range(16):
        out, lse, st = _run(qkv, w, x, cache, q, L - n_q)
        assert st == 0
        _check(out, lse, ro, rl)


def test_prefill_outliers_and_scale(qkv):
    """1 % of K rows x20 (the 1M workload's outliers) and an explicit softmax scale."""
    w, x, ref, cache, q = _setup(qkv, 1200, 96, 64, 16, 4, outliers=0.01, seed=3)
    out, lse, st = _run(qkv, w, x, cache, q, 1104, softmax_scale=0.11)
    assert st == 0
    ro, rl = oracle.prefill_attention(q, ref, x["page_table"][0], np.arange(1104, 1200), 16, 4, 256, 64, 0.11)
    _check(out, lse, ro, rl)


def test_prefill_first_query_is_value(qkv):
    """Query 0 of a chunk with no prefix attends token 0 alone: p = 1, so the
    output is token 0's dequantised value for every head, here rounded to
    fp16 in the tensor-core operand and then to bf16: within one bf16 ulp."""
    w, x, ref, cache, q = _setup(qkv, 70, 70, 16, 16, 4)
    out, _, st = _run(qkv, w, x, cache, q, 0)
    ro, _ = oracle.prefill_attention(q[:1], ref, x["page_table"][0], np.arange(0, 1), 16, 4, 256, 16)
    got = oracle.bf16_to_f64(out[0])
    assert st == 0 and np.all(np.abs(got - ro[0]) <= bf16_ulp(ro[0]))


def test_prefill_bad_page_flagged(qkv):
    w, x, ref, cache, q = _setup(qkv, 200, 50, 64, 16, 4)
    pt = x["page_table"][0].copy()
    pt[1] = w.num_pages + 5
    _, _, st = _run(qkv, w, x, cache, q, 150, page_table=pt)
    assert st == qkv.DEV_BAD_PAGE


def test_prefill_argument_errors(qkv):
    w, x, ref, cache, q = _setup(qkv, 100, 10, 64, 16, 4)
    with pytest.raises(qkv.QkvError) as e:         # prefix + n_q past the page-table row
        _run(qkv, w, x, cache, q, 10 ** 6)
    assert e.value.code == 1
    with pytest.raises(qkv.QkvError) as e:         # 3 parts of a 2-stage context
        _run(qkv, w, x, cache, q, 90, num_splits=3, ws_splits=3)
    assert e.value.code == 1
    with pytest.raises(qkv.QkvError) as e:         # 2 parts without a workspace
        _run(qkv, w, x, cache, q, 90, num_splits=2)
    assert e.value.code == 1
