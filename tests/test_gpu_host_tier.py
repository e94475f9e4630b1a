"""GPU parity of the host-placed K/V tier: qkv_stage_pages_f4 (pages of a
pinned host pool copied into a device window, read in place over the host
link) byte for byte, and qkv_paged_decode_attn_f4_tiered (the older whole
pages of each sequence in the host pool, the rest in the device pool)
against the oracle's attention over the two pools, for several sequences,
windows smaller and larger than the host part, empty tiers, both V scale
layouts and three query-group sizes; and the tiered prefill."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import attn_within, oracle_layer, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _pools(qkv, w, v_group):
    """The workload's cache written on the GPU (device pool) and copied into a
    pinned host pool; the oracle's cache of the same rows."""
    x, ref = oracle_layer(w, v_group=v_group)
    dev = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group)
    dev.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    dev.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    host = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group,
                                     pinned=True)
    for a, b in zip((host.k_data, host.k_scale, host.v_data, host.v_scale),
                    (dev.k_data, dev.k_scale, dev.v_data, dev.v_scale)):
        a.copy_(b)
    torch.cuda.synchronize()
    return x, ref, dev, host


def _split_tables(pt, seq_lens, host_pages, block):
    """First host_pages[s] pages of each row to the host table, the rest to
    the device table."""
    n_seq = len(seq_lens)
    hpt = np.full((n_seq, max(1, max(host_pages))), -1, np.int32)
    dpt = np.full((n_seq, pt.shape[1]), -1, np.int32)
    host_lens, dev_lens = [], []
    for s in range(n_seq):
        h = host_pages[s]
        hpt[s, :h] = pt[s, :h]
        dpt[s, :pt.shape[1] - h] = pt[s, h:]
        host_lens.append(h * block)
        dev_lens.append(int(seq_lens[s]) - h * block)
    return hpt, dpt, np.array(host_lens, np.int32), np.array(dev_lens, np.int32)


CASES = [
    # seq_lens, block, q_heads, kv_heads, num_pages, host pages per sequence, window pages
    ((4096,), 16, 16, 4, 256, (200,), 64),
    ((1000, 31, 4097, 0), 32, 32, 4, 200, (20, 0, 100, 0), 50),
    ((700, 64, 129), 64, 16, 16, 30, (10, 1, 2), 4),
    ((5000, 3000), 64, 16, 8, 140, (78, 46), 200),
    ((2048,), 64, 8, 4, 40, (32,), 7),
]


@pytest.mark.parametrize("v_group", [32, "head_dim"])
@pytest.mark.parametrize("case", CASES + [CASES[1] + (128,)],
                         ids=[f"L{c[0]}-B{c[1]}-G{c[2] // c[3]}-W{c[6]}" + ("-D128" if len(c) > 7 else "")
                              for c in CASES + [CASES[1] + (128,)]])
def test_tiered_decode_matches_oracle(qkv, case, v_group):
    seq_lens, block, hq, hkv, pages, host_pages, window = case[:7]
    head_dim = case[7] if len(case) > 7 else 256
    v_group = head_dim if v_group == "head_dim" else v_group
    w = workloads.small("tier", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous", head_scale=True,
                        head_dim=head_dim)
    x, ref, dev, host = _pools(qkv, w, v_group)
    hpt, dpt, host_lens, dev_lens = _split_tables(x["page_table"], x["seq_lens"], host_pages, block)
    att = qkv.TieredDecodeAttention(hq, hkv, w.head_dim, block, hpt.shape[1], window, v_group=v_group)
    out = torch.empty((w.n_seq, hq, w.head_dim), dtype=torch.int16, device="cuda")
    lse = torch.empty((w.n_seq, hq), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    att(out, to_dev(x["q"]), dev, to_dev(dpt), to_dev(dev_lens), host, torch.from_numpy(hpt).pin_memory(),
        host_lens, lse2_out=lse, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.tiered_attention(x["q"], ref, hpt, host_lens, ref, dpt, dev_lens, hq, hkv, w.head_dim, block)
    got = to_host(out, np.uint16)
    lg = to_host(lse)
    for s in range(w.n_seq):
        if host_lens[s] + dev_lens[s] == 0:  # empty context: zero output, lse2 -inf
            assert np.all(got[s] == 0) and np.all(np.isneginf(lg[s]))
            continue
        err, bound = attn_within(got[s], ro[s])
        assert np.all(err <= bound), f"seq {s}: max err {err.max():.3e}"
        assert np.max(np.abs(lg[s] - rl[s])) <= 2e-4


def test_tiered_all_on_host_equals_device_decode(qkv):
    """The whole context in the host tier (device parts empty) against the
    one-pool decode of the same cache: both within tolerance of the oracle
    and of each other."""
    w = workloads.small("tier_all", seq_lens=(3072, 1024), num_pages=64, block_size=64, page_alloc="interleaved")
    x, ref, dev, host = _pools(qkv, w, 32)
    hpt, dpt, host_lens, dev_lens = _split_tables(x["page_table"], x["seq_lens"], (48, 16), 64)
    assert np.all(dev_lens == 0)
    att = qkv.TieredDecodeAttention(w.q_heads, w.kv_heads, w.head_dim, 64, hpt.shape[1], 16)
    out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
    att(out, to_dev(x["q"]), dev, to_dev(dpt), to_dev(dev_lens), host, to_dev(hpt), host_lens)
    one = torch.empty_like(out)
    qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, 64)(
        one, to_dev(x["q"]), dev, to_dev(x["page_table"]), to_dev(x["seq_lens"]))
    torch.cuda.synchronize()
    ro, _ = oracle.paged_attention(x["q"], ref, x["page_table"], np.zeros(w.n_seq, np.int32), x["seq_lens"],
                                   w.q_heads, w.kv_heads, w.head_dim, 64)
    for t in (out, one):
        err, bound = attn_within(to_host(t, np.uint16), ro)
        assert np.all(err <= bound)


@pytest.mark.parametrize("v_group", [32, 128])
@pytest.mark.parametrize("source", ["pinned", "device"])
def test_stage_pages_bitexact(qkv, source, v_group):
    rng = np.random.default_rng(21)
    pages, hkv, block, d = 40, 2, 32, 128
    src = qkv.PagedF4Cache.allocate(pages, hkv, block, d, v_group=v_group, pinned=(source == "pinned"))
    for t in (src.k_data, src.v_data):
        t.copy_(torch.from_numpy(rng.integers(0, 256, size=t.shape, dtype=np.uint8)))
    for t in (src.k_scale, src.v_scale):
        t.copy_(torch.from_numpy(rng.integers(0, 1 << 15, size=t.shape, dtype=np.int16)).view(torch.float16))
    win = qkv.PagedF4Cache.allocate(30, hkv, block, d, v_group=v_group)
    for t in (win.k_data, win.k_scale, win.v_data, win.v_scale):
        t.view(torch.uint8).fill_(0xA5)
    ids = rng.integers(0, pages, size=12).astype(np.int32)
    ids[3] = ids[7]                                               # a page staged twice
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_stage_pages_f4(win.k_data, win.k_scale, win.v_data, win.v_scale, src.k_data, src.k_scale, src.v_data,
                           src.v_scale, to_dev(ids), dst_page0=5, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for a, b in zip((win.k_data, win.k_scale, win.v_data, win.v_scale),
                    (src.k_data, src.k_scale, src.v_data, src.v_scale)):
        got = a.cpu().view(torch.uint8).numpy()
        want = b.cpu().view(torch.uint8).numpy()
        assert np.array_equal(got[5:17], want[ids])
        assert np.all(got[:5] == 0xA5) and np.all(got[17:] == 0xA5)  # nothing else written


def test_stage_bad_page_zero_fills_and_flags(qkv):
    src = qkv.PagedF4Cache.allocate(8, 4, 64, 256, pinned=True)
    src.k_data.fill_(0x33)
    win = qkv.PagedF4Cache.allocate(4, 4, 64, 256)
    win.k_data.fill_(0x77)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ids = torch.tensor([1, 8, -1, 2], dtype=torch.int32, device="cuda")
    qkv.qkv_stage_pages_f4(win.k_data, win.k_scale, win.v_data, win.v_scale, src.k_data, src.k_scale, src.v_data,
                           src.v_scale, ids, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == qkv.DEV_BAD_PAGE
    k = win.k_data.cpu().numpy()
    assert np.all(k[[0, 3]] == 0x33) and np.all(k[[1, 2]] == 0)


def test_pageable_host_memory_refused_on_host(qkv):
    """A pageable host pointer is refused before any launch (the call asks the
    driver what each source pointer is)."""
    import ctypes
    win = qkv.PagedF4Cache.allocate(2, 4, 64, 256)
    pageable = torch.zeros(8 * 4 * 64 * 128, dtype=torch.uint8)          # not pinned
    assert not pageable.is_pinned()
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptr = ctypes.c_void_p(pageable.data_ptr())
    rc = qkv.lib.qkv_stage_pages_f4(win.k_data.data_ptr(), win.k_scale.data_ptr(), win.v_data.data_ptr(),
                                    win.v_scale.data_ptr(), 2, 0, ptr, ptr, ptr, ptr, 8, ids.data_ptr(), 1, 4, 256, 64,
                                    32, None, None)
    assert rc == 1
    with pytest.raises(ValueError):
        qkv.qkv_stage_pages_f4(win.k_data, win.k_scale, win.v_data, win.v_scale, pageable.view(8, 4, 64, 128),
                               win.k_scale, win.v_data, win.v_scale, ids)


PF_CASES = [
    # host pages, device tokens (prefix + chunk), chunk, block, q_heads, kv_heads, window pages, parts per launch
    (40, 700, 300, 16, 16, 4, 16, 4),     # ragged chunk and prefix, three windows (16, 16, 8)
    (8, 130, 130, 64, 8, 8, 3, 2),        # the chunk is the whole device part, G = 1, windows 3, 3, 2
    (0, 1000, 257, 32, 32, 4, 4, 4),      # no host part, G = 8
    (20, 64, 1, 64, 16, 4, 64, 8),        # one query, the window larger than the host part
    (30, 500, 200, 16, 16, 4, 12, 4, 128),  # head_dim 128
]


@pytest.mark.parametrize("v_group", [32, "head_dim"])
@pytest.mark.parametrize("case", PF_CASES, ids=[f"H{c[0]}-L{c[1]}-Q{c[2]}-B{c[3]}-W{c[6]}" +
                                                ("-D128" if len(c) > 8 else "") for c in PF_CASES])
def test_tiered_prefill_matches_oracle(qkv, case, v_group):
    hp, dev_tokens, n_q, block, hq, hkv, window, ppl = case[:8]
    d = case[8] if len(case) > 8 else 256
    v_group = d if v_group == "head_dim" else v_group
    ctx = hp * block + dev_tokens
    w = workloads.small("tier_pf", seq_lens=(ctx,), num_pages=-(-ctx // block) + 2, block_size=block, q_heads=hq,
                        kv_heads=hkv, head_scale=True, head_dim=d)
    x, ref, dev, host = _pools(qkv, w, v_group)
    row = x["page_table"][0]
    hrow, drow = np.ascontiguousarray(row[:max(hp, 1)]), np.ascontiguousarray(row[hp:])
    prefix = dev_tokens - n_q
    q = workloads.chunk_queries_host(w, 0, n_q)
    att = qkv.TieredPrefillAttention(n_q, hq, hkv, d, block, hp, window, v_group=v_group, parts_per_launch=ppl)
    out = torch.full((n_q, hq, d), 0x7FC1, dtype=torch.int16, device="cuda")
    lse = torch.empty((n_q, hq), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    att(out, to_dev(q), dev, to_dev(drow), prefix, host, torch.from_numpy(hrow).pin_memory(), hp * block,
        lse2_out=lse, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ro, rl = oracle.tiered_prefill_attention(q, ref, hrow, hp * block, ref, drow, np.arange(prefix, dev_tokens), hq,
                                             hkv, d, block)
    err, bound = attn_within(to_host(out, np.uint16), ro)
    assert np.all(err <= bound), f"max err {err.max():.3e} (excess {np.max(err - bound):.3e})"
    assert np.max(np.abs(to_host(lse) - rl)) <= 2e-3


def test_tiered_prefill_equals_one_pool_prefill(qkv):
    """The same chunk with its first 24 pages in the host tier and with the
    whole context in the device pool: both within tolerance of the oracle."""
    w = workloads.small("tier_pf1", seq_lens=(2000,), num_pages=40, block_size=64, head_scale=True)
    x, ref, dev, host = _pools(qkv, w, 32)
    row = x["page_table"][0]
    n_q, hp = 200, 24
    q = workloads.chunk_queries_host(w, 0, n_q)
    nb = qkv.qkv_paged_prefill_tiered_workspace_bytes(n_q, w.q_heads, w.kv_heads, 256, 64, 32, hp, 10, 4)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    a = torch.empty((n_q, w.q_heads, 256), dtype=torch.int16, device="cuda")
    qkv.qkv_paged_prefill_attn_f4_tiered(a, to_dev(q), dev.k_data, dev.k_scale, dev.v_data, dev.v_scale,
                                         to_dev(np.ascontiguousarray(row[hp:])), 2000 - hp * 64 - n_q, host.k_data,
                                         host.k_scale, host.v_data, host.v_scale, to_dev(np.ascontiguousarray(row[:hp])),
                                         hp * 64, w.kv_heads, 10, 4, ws)
    b = torch.empty_like(a)
    qkv.qkv_paged_prefill_attn_f4(b, to_dev(q), dev.k_data, dev.k_scale, dev.v_data, dev.v_scale, to_dev(row),
                                  2000 - n_q, w.kv_heads)
    torch.cuda.synchronize()
    ro, _ = oracle.prefill_attention(q, ref, row, np.arange(2000 - n_q, 2000), w.q_heads, w.kv_heads, 256, 64)
    for t in (a, b):
        err, bound = attn_within(to_host(t, np.uint16), ro)
        assert np.all(err <= bound)
