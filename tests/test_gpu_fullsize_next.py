"""Parity of the gather and the chunked prefill at the bench's full size
(the yarn262k layer-0 cache: 262,144 tokens, 4 KV heads), in the launch
configuration `bench.py --op gather|prefill` times.

Gather: the whole context's bf16 K/V rows against the oracle's gather, bit
for bit. Prefill: the 2048-query chunk at the end of the context on the GPU;
the oracle's exact causal attention for a sample of queries (first, last and
spread between) and all 16 heads, within the attention tolerance."""
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


@pytest.fixture(scope="module")
def layer(qkv):
    """yarn262k layer 0 on the GPU (all 262,144 tokens written) and its
    oracle cache from the same generated bf16 rows."""
    w = workloads.YARN_262K
    dev = torch.device("cuda:0")
    x = workloads.device_layer(w, 0, dev)
    cache = qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    cache.write(x["k_cache"], x["v_cache"], x["cache_slots"])
    cache.write(x["k_new"], x["v_new"], x["step_slots"])
    h = {k: to_host(v, np.uint16) if v.dtype == torch.int16 else to_host(v)
         for k, v in x.items() if isinstance(v, torch.Tensor)}
    ref = oracle.empty_cache(w.num_pages, w.kv_heads, w.block_size, w.head_dim)
    assert oracle.kv_write_f4(h["k_cache"], h["v_cache"], h["cache_slots"], ref, w.kv_heads, w.head_dim,
                              w.block_size) == 0
    assert oracle.kv_write_f4(h["k_new"], h["v_new"], h["step_slots"], ref, w.kv_heads, w.head_dim,
                              w.block_size) == 0
    return w, x, h, cache, ref


def test_fullsize_gather(qkv, layer):
    w, x, h, cache, ref = layer
    ctx = int(w.seq_lens[0])
    k_out = torch.empty((ctx, w.kv_heads, w.head_dim), dtype=torch.int16, device="cuda")
    v_out = torch.empty_like(k_out)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    start = torch.zeros(1, dtype=torch.int64, device="cuda")
    qkv.qkv_gather_kv_f4(k_out, v_out, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, x["page_table"],
                         x["seq_lens"], start, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rk, rv, bad = oracle.gather_kv_f4(ref, h["page_table"], h["seq_lens"], [0], w.kv_heads, w.head_dim,
                                      w.block_size)
    assert bad == 0
    assert np.array_equal(to_host(k_out, np.uint16), rk)
    assert np.array_equal(to_host(v_out, np.uint16), rv)


def test_fullsize_prefill_sampled(qkv, layer):
    w, x, h, cache, ref = layer
    ctx, n_q = int(w.seq_lens[0]), 2048
    prefix = ctx - n_q
    q = workloads.chunk_queries_device(w, 0, n_q, torch.device("cuda:0"))
    out = torch.empty_like(q)
    lse = torch.empty((n_q, w.q_heads), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_paged_prefill_attn_f4(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                                  x["page_table"][0].contiguous(), prefix, w.kv_heads, lse2_out=lse,
                                  device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    pick = np.array([0, 1, 255, 256, 1023, 1024, 1800, n_q - 1])
    qh = to_host(q, np.uint16)[pick]
    ro, rl = oracle.prefill_attention(qh, ref, h["page_table"][0], prefix + pick, w.q_heads, w.kv_heads,
                                      w.head_dim, w.block_size)
    err, bound = attn_within(to_host(out, np.uint16)[pick], ro)
    assert np.all(err <= bound), f"max err {err.max():.3e}, worst excess {np.max(err - bound):.3e}"
    assert np.max(np.abs(to_host(lse)[pick] - rl)) <= 2e-3
