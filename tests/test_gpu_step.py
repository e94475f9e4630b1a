"""The fused decode step (qkv_decode_step_f4: rotary and F4 write of the new
token inside the split launch, then the merge) gives the same bits as the
two-call path qkv_rope_kv_write_f4 + qkv_paged_decode_attn_f4 -- outputs,
lse2 and the whole cache -- whose oracle parity the other GPU tests pin.
One case is also checked against the oracle directly."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import attn_within, oracle_layer, to_dev, to_host

pytestmark = pytest.mark.gpu

YARN4 = dict(rope_base=1e7, rot_dim=64, factor=4.0, orig_max_pos=262144, beta_fast=32.0, beta_slow=1.0)


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _table(qkv, spec, pos0, n):
    h = spec["rot_dim"] // 2
    c = torch.empty((n, h), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    qkv.qkv_yarn_rope_table(qkv.YarnParams.make(**spec), pos0, n, c, s)
    return c, s


def _both(qkv, w, x, v_group, spec, num_splits=0, positions=None, slots=None, table=None):
    """Run the two-call path and the fused step on identical caches."""
    pos = x["positions"] if positions is None else positions
    slots = x["step_slots"] if slots is None else slots
    p0 = int(np.min(x["positions"])) - 3
    c, s = table if table is not None else _table(qkv, spec, p0, int(np.max(x["positions"])) - p0 + 4)
    caches = []
    for _ in range(2):
        cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group)
        cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
        caches.append(cache)
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size,
                              max_splits=max(40, num_splits))
    outs = []
    # two calls
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q_rot = torch.empty_like(to_dev(x["q"]))
    ca = caches[0]
    qkv.qkv_rope_kv_write_f4(to_dev(x["q"]), q_rot, to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(pos),
                             to_dev(slots), c, s, p0, spec["rot_dim"], ca.k_data, ca.k_scale, ca.v_data, ca.v_scale,
                             device_status=st)
    out = torch.empty_like(q_rot)
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
    att(out, q_rot, ca, to_dev(x["page_table"]), to_dev(x["seq_lens"]), lse2_out=lse, num_splits=num_splits,
        device_status=st)
    outs.append((to_host(out, np.uint16), to_host(lse), int(st.item())))
    # the fused step
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cb = caches[1]
    out = torch.empty_like(q_rot)
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
    att.step(out, to_dev(x["q"]), to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(pos), to_dev(slots), c, s, p0,
             spec["rot_dim"], cb, to_dev(x["page_table"]), to_dev(x["seq_lens"]), lse2_out=lse,
             num_splits=num_splits, device_status=st)
    outs.append((to_host(out, np.uint16), to_host(lse), int(st.item())))
    return outs, caches


def _same_cache(a, b):
    for ta, tb in zip((a.k_data, a.k_scale, a.v_data, a.v_scale), (b.k_data, b.k_scale, b.v_data, b.v_scale)):
        assert torch.equal(ta, tb)


CASES = [
    # seq_lens, block, q_heads, kv_heads, num_pages, num_splits
    ((4096,), 16, 16, 4, 256, 4),
    ((1, 2, 15, 16, 17), 16, 16, 4, 16, 3),
    ((63, 64, 65, 127, 129), 64, 8, 2, 16, 2),
    ((1000, 31, 4097, 0, 1), 32, 32, 4, 200, 0),
    ((700, 1), 32, 16, 16, 30, 100),
    ((5000, 3000, 10), 64, 16, 4, 140, 0),
]


@pytest.mark.parametrize("v_group", [32, 256])
@pytest.mark.parametrize("case", CASES, ids=[f"L{c[0]}-B{c[1]}-G{c[2] // c[3]}-S{c[5]}" for c in CASES])
def test_step_matches_two_calls(qkv, case, v_group):
    seq_lens, block, hq, hkv, pages, splits = case
    w = workloads.small("step", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous", head_scale=True,
                        yarn_factor=4.0, first_position=300000)
    x = workloads.host_layer(w)
    outs, caches = _both(qkv, w, x, v_group, YARN4, num_splits=splits)
    (oa, la, sa), (ob, lb, sb) = outs
    assert sa == 0 and sb == 0
    assert np.array_equal(oa, ob)
    assert np.array_equal(la.view(np.uint32), lb.view(np.uint32))
    _same_cache(*caches)


@pytest.mark.parametrize("v_group", [32, 128])
@pytest.mark.parametrize("case", [((4096,), 16, 16, 4, 256, 4), ((63, 64, 65, 127, 129), 64, 8, 2, 16, 2),
                                  ((1000, 31, 4097, 0, 1), 32, 32, 4, 200, 0)],
                         ids=["L4096-B16-G4", "L5-B64-G4", "L5-B32-G8"])
def test_step_matches_two_calls_head_dim_128(qkv, case, v_group):
    seq_lens, block, hq, hkv, pages, splits = case
    w = workloads.small("step128", seq_lens=seq_lens, num_pages=pages, block_size=block, q_heads=hq, kv_heads=hkv,
                        head_dim=128, page_alloc="interleaved" if len(seq_lens) > 1 else "contiguous",
                        head_scale=True, yarn_factor=4.0, first_position=300000)
    x = workloads.host_layer(w)
    outs, caches = _both(qkv, w, x, v_group, YARN4, num_splits=splits)
    (oa, la, sa), (ob, lb, sb) = outs
    assert sa == 0 and sb == 0
    assert np.array_equal(oa, ob)
    assert np.array_equal(la.view(np.uint32), lb.view(np.uint32))
    _same_cache(*caches)


@pytest.mark.parametrize("head_dim", [256, 128])
def test_step_matches_oracle(qkv, head_dim):
    """rotary (oracle) -> F4 write (oracle) -> exact attention (oracle)."""
    w = workloads.small("step_o", seq_lens=(3000, 70, 1), num_pages=64, block_size=64, head_scale=True,
                        page_alloc="interleaved", yarn_factor=4.0, first_position=400000, head_dim=head_dim)
    x = workloads.host_layer(w)
    outs, caches = _both(qkv, w, x, 32, YARN4)
    ob, lb, sb = outs[1]
    assert sb == 0
    spec = workloads.yarn_spec(w)
    q = oracle.rope_apply_bf16(x["q"], x["positions"], spec)
    k = oracle.rope_apply_bf16(x["k_new"], x["positions"], spec)
    ref = oracle.empty_cache(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    oracle.kv_write_f4(x["k_cache"], x["v_cache"], x["cache_slots"], ref, w.kv_heads, w.head_dim, w.block_size)
    oracle.kv_write_f4(k, x["v_new"], x["step_slots"], ref, w.kv_heads, w.head_dim, w.block_size)
    got = (to_host(caches[1].k_data), to_host(caches[1].k_scale).view(np.uint16), to_host(caches[1].v_data),
           to_host(caches[1].v_scale).view(np.uint16))
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)
    ro, rl = oracle.paged_attention(q, ref, x["page_table"], np.zeros(w.n_seq, np.int32), x["seq_lens"], w.q_heads,
                                    w.kv_heads, w.head_dim, w.block_size)
    err, bound = attn_within(ob, ro)
    assert np.all(err <= bound)
    assert np.max(np.abs(lb - rl)) <= 2e-4


def test_step_flags(qkv):
    w = workloads.small("step_f", seq_lens=(100, 64), num_pages=4, block_size=64, yarn_factor=4.0,
                        first_position=300000)
    x = workloads.host_layer(w)
    c, s = _table(qkv, YARN4, 300000, 10)             # positions 300099, 300063 lie outside
    outs, caches = _both(qkv, w, x, 32, YARN4, table=(c, s))
    assert outs[0][2] == outs[1][2] == qkv.DEV_BAD_POSITION
    assert np.array_equal(outs[0][0], outs[1][0])
    _same_cache(*caches)
    slots = x["step_slots"].copy()
    slots[1] = w.num_pages * w.block_size + 3           # past the pool: write skipped, flagged
    outs, caches = _both(qkv, w, x, 32, YARN4, slots=slots)
    assert outs[0][2] == outs[1][2] == qkv.DEV_BAD_SLOT
    assert np.array_equal(outs[0][0], outs[1][0])
    _same_cache(*caches)
