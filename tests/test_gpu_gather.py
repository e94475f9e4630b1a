"""GPU parity of the paged F4 gather (qkv_gather_kv_f4) with the oracle:
bit-exact bf16 rows for several sequences sharing one interleaved pool,
ragged lengths, an empty sequence, both V scale layouts and three head
sizes; bad page ids and lengths are flagged."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import oracle_layer, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _setup(qkv, w, v_group):
    x, ref = oracle_layer(w, v_group=v_group)
    cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group)
    cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    cache.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    return x, ref, cache


def _gather(qkv, w, cache, page_table, seq_lens, start, n_out):
    ko = torch.full((n_out, w.kv_heads, w.head_dim), 0x7FC1, dtype=torch.int16, device="cuda")
    vo = torch.full_like(ko, 0x7FC1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_gather_kv_f4(ko, vo, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, to_dev(page_table),
                         to_dev(np.asarray(seq_lens, np.int32)), to_dev(np.asarray(start, np.int64)),
                         device_status=st)
    return to_host(ko, np.uint16), to_host(vo, np.uint16), int(st.item())


CASES = [
    # seq_lens, block, head_dim, kv_heads, num_pages
    ((1000, 0, 31, 4097), 32, 256, 4, 200),
    ((700, 64, 65), 64, 128, 2, 40),
    ((129, 16), 16, 64, 4, 20),
]


@pytest.mark.parametrize("v_group", [32, 0])
@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-B{c[1]}-D{c[2]}" for c in CASES])
def test_gather_bitexact(qkv, case, v_group):
    seq_lens, block, d, hkv, pages = case
    v_group = v_group or d
    w = workloads.small("gather", seq_lens=seq_lens, num_pages=pages, block_size=block, head_dim=d,
                        q_heads=hkv * 4, kv_heads=hkv, page_alloc="interleaved", head_scale=True)
    x, ref, cache = _setup(qkv, w, v_group)
    lens = np.asarray(x["seq_lens"], np.int32)
    start = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64) + 3   # a gap before the first row
    n_out = int(start[-1] + lens[-1]) + 2
    ko, vo, st = _gather(qkv, w, cache, x["page_table"], lens, start, n_out)
    assert st == 0
    rk, rv, bad = oracle.gather_kv_f4(ref, x["page_table"], lens, start, w.kv_heads, d, block, n_out)
    assert bad == 0
    for s, L in enumerate(lens):
        rows = slice(start[s], start[s] + L)
        assert np.array_equal(ko[rows], rk[rows]) and np.array_equal(vo[rows], rv[rows])
    # rows outside every sequence are left as they were
    written = np.zeros(n_out, bool)
    for s, L in enumerate(lens):
        written[start[s]:start[s] + L] = True
    assert np.all(ko[~written] == 0x7FC1) and np.all(vo[~written] == 0x7FC1)


def test_gather_flags(qkv):
    w = workloads.small("gflag", seq_lens=(100, 64), num_pages=4, block_size=64, head_dim=256, q_heads=16,
                        kv_heads=4)
    x, ref, cache = _setup(qkv, w, 32)
    lens = np.asarray(x["seq_lens"], np.int32)
    pt = x["page_table"].copy()
    pt[0, 1] = 99                                   # page id outside the pool: tokens 64..99 of sequence 0
    ko, vo, st = _gather(qkv, w, cache, pt, lens, [0, 100], 164)
    assert st == qkv.DEV_BAD_PAGE
    rk, rv, bad = oracle.gather_kv_f4(ref, pt, lens, [0, 100], w.kv_heads, 256, 64, 164)
    assert bad == 36
    assert np.array_equal(ko, rk) and np.array_equal(vo, rv)
    # clamped to the 128 tokens of its page-table row, whose second page is unused (-1)
    _, _, st = _gather(qkv, w, cache, x["page_table"], np.array([100, 10 ** 6], np.int32), [0, 100], 10 ** 4)
    assert st == qkv.DEV_BAD_SEQLEN | qkv.DEV_BAD_PAGE
    _, _, st = _gather(qkv, w, cache, x["page_table"], lens, [0, 150], 164)     # sequence 1 overruns n_out
    assert st == qkv.DEV_BAD_SEQLEN
