"""Decode attention through the entry point that allocates nothing.

Some callers can't call cudaMalloc -- a plugin running inside a host engine
that owns all device memory, or a runtime whose memory budget is fixed at
start-up -- so they cannot hand the library a partials workspace.
qkv_paged_decode_attn_f4_static keeps the partials in an array compiled into
the library instead. These tests call it through the C ABI and check it
against the workspace entry point, twice in a row on different inputs (the
array keeps the previous call's contents), and check that a problem too large
for the array is refused."""
import numpy as np
import pytest
import torch

import workloads
from helpers import attn_within, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _inputs(qkv, w):
    x = workloads.host_layer(w)
    cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    cache.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    return x, cache


def _outputs(w):
    out = torch.empty((w.n_seq, w.q_heads, w.head_dim), dtype=torch.int16, device="cuda")
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device="cuda")
    return out, lse


CALLS = [
    workloads.small("noalloc_a", seq_lens=(3000, 1000, 17), num_pages=80, block_size=64, head_scale=True),
    workloads.small("noalloc_b", seq_lens=(5000,), num_pages=320, block_size=16, q_heads=8, kv_heads=4, seed=7),
]


def test_static_scratch_matches_workspace_entry_point(qkv):
    for w in CALLS:  # two calls in a row through the shared array
        x, cache = _inputs(qkv, w)
        q, pt, sl = to_dev(x["q"]), to_dev(x["page_table"]), to_dev(x["seq_lens"])
        st = torch.zeros(1, dtype=torch.int32, device="cuda")

        ref_out, ref_lse = _outputs(w)
        att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size)
        att(ref_out, q, cache, pt, sl, lse2_out=ref_lse, device_status=st)

        out, lse = _outputs(w)
        out.fill_(-1)
        lse.fill_(float("nan"))
        qkv.qkv_paged_decode_attn_f4_static(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, pt,
                                            sl, w.kv_heads, lse2_out=lse, device_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0

        ref = workloads.bf16_bits_to_f32(to_host(ref_out, np.uint16)).astype(np.float64)
        err, bound = attn_within(to_host(out, np.uint16), ref)
        assert np.all(err <= bound), f"{w.name}: max err {err.max():.3e}"
        got_l, ref_l = to_host(lse), to_host(ref_lse)
        assert np.all(np.isfinite(got_l))
        assert np.max(np.abs(got_l - ref_l)) <= 2e-4


def test_static_scratch_refuses_oversize(qkv):
    w = workloads.small("noalloc_big", seq_lens=(64,) * 4, num_pages=8, block_size=64)
    x, cache = _inputs(qkv, w)
    out, lse = _outputs(w)
    need = qkv.qkv_paged_decode_workspace_bytes(w.n_seq, w.q_heads, w.head_dim, 400)
    assert need > qkv.STATIC_SCRATCH_BYTES
    with pytest.raises(qkv.QkvError) as e:
        qkv.qkv_paged_decode_attn_f4_static(out, to_dev(x["q"]), cache.k_data, cache.k_scale, cache.v_data,
                                            cache.v_scale, to_dev(x["page_table"]), to_dev(x["seq_lens"]),
                                            w.kv_heads, num_splits=400)
    assert e.value.code == 1
