"""Parity at the workloads' full sizes, in the launch configuration the bench
times (automatic split plan, all heads), on layer 0 of each workload.

Inputs come from the device generator; the oracle gets the same bf16 arrays
copied to the host. Checked: the whole layer's F4 cache bit for bit, and the
attention output of every (sequence, query head) row within the attention
tolerance. The decode step's rotary and write of the new token use the fused
call, as the bench does."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import attn_within, to_host

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


@pytest.mark.parametrize("name", [w.name for w in workloads.ALL])
def test_fullsize_layer0(qkv, name):
    w = workloads.BY_NAME[name]
    dev = torch.device("cuda:0")
    x = workloads.device_layer(w, 0, dev)
    cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    cache.write(x["k_cache"], x["v_cache"], x["cache_slots"], device_status=st)
    # decode step: table rows of the step positions, fused rotary + write, attention
    pos = w.step_positions
    p0, n_rows = min(pos), max(pos) - min(pos) + 1
    cos = torch.empty((n_rows, w.rot_dim // 2), dtype=torch.float32, device=dev)
    sin = torch.empty_like(cos)
    qkv.qkv_yarn_rope_table(qkv.YarnParams.make(**workloads.yarn_spec(w)), p0, n_rows, cos, sin)
    q_rot = torch.empty_like(x["q"])
    k_rot = torch.empty_like(x["k_new"])
    qkv.qkv_rope_kv_write_f4(x["q"], q_rot, x["k_new"], x["v_new"], x["positions"], x["step_slots"], cos, sin, p0,
                             w.rot_dim, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, k_out=k_rot,
                             device_status=st)
    # the workload's own split plan: a fixed count sizes the workspace (148 at
    # 1,048,576 tokens), otherwise the automatic plan
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size, max_splits=w.num_splits)
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.n_seq, w.q_heads), dtype=torch.float32, device=dev)
    att(out, q_rot, cache, x["page_table"], x["seq_lens"], lse2_out=lse, num_splits=w.num_splits, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    _, l_parts = att.partials(w.n_seq, w.q_heads, w.head_dim)
    weighted = np.isfinite(to_host(l_parts)).sum(0)       # parts merged per query row
    if w.num_splits:
        assert att.max_splits == w.num_splits
        assert np.all(weighted == w.num_splits), weighted
    else:
        assert np.all(weighted >= 1)

    # oracle: the same generated inputs, on the host
    h = {k: to_host(v, np.uint16) if v.dtype == torch.int16 else to_host(v)
         for k, v in x.items() if isinstance(v, torch.Tensor)}
    spec = workloads.yarn_spec(w)
    q_ref = oracle.rope_apply_bf16(h["q"], h["positions"], spec)
    k_ref = oracle.rope_apply_bf16(h["k_new"], h["positions"], spec)
    ref = oracle.empty_cache(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    assert oracle.kv_write_f4(h["k_cache"], h["v_cache"], h["cache_slots"], ref, w.kv_heads, w.head_dim,
                              w.block_size) == 0
    # the context cache is bit-exact
    got = (to_host(cache.k_data), to_host(cache.k_scale).view(np.uint16), to_host(cache.v_data),
           to_host(cache.v_scale).view(np.uint16))
    step_rows = np.zeros(got[0].shape[:3], bool)
    for slot in h["step_slots"]:
        step_rows[slot // w.block_size, :, slot % w.block_size] = True
    for a, b in zip(got, ref):
        assert np.array_equal(a[~step_rows], b[~step_rows])
    # the new token: the GPU's rotary is within one bf16 step of the oracle's; the oracle then writes
    # the token from its own rotary
    qd = np.abs(workloads.bf16_bits_to_f32(to_host(q_rot, np.uint16)).astype(np.float64) - oracle.bf16_to_f64(q_ref))
    assert np.all(qd <= np.abs(oracle.bf16_to_f64(q_ref)) * 2.0 ** -7 + 1e-30)
    assert oracle.kv_write_f4(k_ref, h["v_new"], h["step_slots"], ref, w.kv_heads, w.head_dim, w.block_size) == 0
    ro, rl = oracle.paged_attention(q_ref, ref, h["page_table"], np.zeros(w.n_seq, np.int32), h["seq_lens"],
                                    w.q_heads, w.kv_heads, w.head_dim, w.block_size)
    err, bound = attn_within(to_host(out, np.uint16), ro)
    assert np.all(err <= bound), f"{name}: max err {err.max():.3e}, worst excess {np.max(err - bound):.3e}"
    assert np.max(np.abs(to_host(lse) - rl)) <= 2e-4
