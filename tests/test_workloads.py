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
