"""The seeded input generators are shared by both sides of every parity test,
so their bookkeeping is checked here: one pre-filled K/V row per cache slot,
one step slot per sequence, and empty contexts handled."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("seq_lens", [(1000, 31, 4097, 0, 1), (0,), (1,), (64, 65, 0)])
def test_rows_match_slots(seq_lens):
    w = workloads.small("gen", seq_lens=seq_lens, num_pages=200, block_size=32, page_alloc="interleaved")
    x = workloads.host_layer(w)
    T = sum(max(L - 1, 0) for L in seq_lens)
    assert x["k_cache"].shape[0] == x["v_cache"].shape[0] == x["cache_slots"].shape[0] == T
    assert x["k_new"].shape[0] == x["step_slots"].shape[0] == x["positions"].shape[0] == len(seq_lens)
    pt = x["page_table"]
    for s, L in enumerate(seq_lens):
        if L == 0:
            assert x["step_slots"][s] == -1
            assert x["positions"][s] == w.first_position
        else:
            page, off = divmod(int(x["step_slots"][s]), w.block_size)
            assert page == pt[s, (L - 1) // w.block_size] and off == (L - 1) % w.block_size
    # every slot is distinct and lies in a page of its own sequence
    slots = np.concatenate([x["cache_slots"], x["step_slots"][x["step_slots"] >= 0]])
    assert len(np.unique(slots)) == len(slots)


def test_binding_rejects_mismatched_slot_mapping():
    torch = pytest.importorskip("torch")
    try:
        from quantized_paged_kv_yarn_b200 import _abi
    except ImportError:
        pytest.skip("library not built")
    k = torch.zeros((5, 4, 256), dtype=torch.int16)
    cache = [torch.zeros((8, 4, 64, 128), dtype=torch.uint8), torch.zeros((8, 4, 64, 8), dtype=torch.int16),
             torch.zeros((8, 4, 64, 128), dtype=torch.uint8), torch.zeros((8, 4, 64, 8), dtype=torch.int16)]
    with pytest.raises(ValueError):
        _abi.qkv_kv_write_f4(k, k, torch.zeros(6, dtype=torch.int64), *cache)


def test_split_plan_as_stated():
    """The split boundaries the GPU tests expect (the plan include/qkv.h
    states): they start at 0, end at n, never decrease, keep splits equal
    below 8 splits, and from 8 on make the first ceil(S/7) splits shorter than
    the rest by the stated amount (at most a quarter split)."""
    from helpers import split_bound
    for n in (1, 7, 57, 118, 2048, 4096, 16384):
        for S in (1, 3, 7, 8, 9, 37, 100, 148):
            for block in (16, 32, 64):
                for hd in (256, 128):
                    b = [split_bound(i, n, S, block, hd) for i in range(S + 1)]
                    assert b[0] == 0 and b[-1] == n
                    assert all(b[i] <= b[i + 1] for i in range(S))
                    sizes = [b[i + 1] - b[i] for i in range(S)]
                    if S < 8:
                        assert max(sizes) - min(sizes) <= 1
                    else:
                        m = (S + 6) // 7
                        d = min((400 if hd == 256 else 800) // block, n // S // 4)
                        if d:
                            assert max(sizes[:m]) < min(sizes[m:])
                            assert sum(sizes[:m]) <= m * (n // S) - m * d + m
    # the 262,144-token workload's plan: 6 of 37 splits ~6 pages shorter per KV head
    sizes = [split_bound(i + 1, 4096, 37, 64, 256) - split_bound(i, 4096, 37, 64, 256) for i in range(37)]
    assert sizes[:6] == [104, 105, 105, 104, 105, 105] and min(sizes[6:]) >= 111
