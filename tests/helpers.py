"""Shared test helpers: building oracle-side caches from the seeded workloads.
(Test infrastructure; uses the oracle and the generator only.)"""
import numpy as np

import oracle
import workloads


def oracle_layer(w, layer=0, inputs=None, with_step=True, v_group=32):
    """Quantise a workload layer into an oracle cache. Returns (inputs, cache).
    With ``with_step`` the decode step's (unroped) k_new/v_new are written too,
    at the step slots; rotary is the caller's business. ``v_group`` picks the
    V scale layout (32 per cell, head_dim per token)."""
    x = inputs if inputs is not None else workloads.host_layer(w, layer)
    cache = oracle.empty_cache(w.num_pages, w.kv_heads, w.block_size, w.head_dim, v_group=v_group)
    bad = oracle.kv_write_f4(x["k_cache"], x["v_cache"], x["cache_slots"], cache, w.kv_heads, w.head_dim,
                             w.block_size)
    assert bad == 0
    if with_step:
        bad = oracle.kv_write_f4(x["k_new"], x["v_new"], x["step_slots"], cache, w.kv_heads, w.head_dim,
                                 w.block_size)
        assert bad == 0
    return x, cache


def dense_dequant(cache, page_table, seq, n_tok, block_size):
    """[n_tok][Hkv][D] float64 K and V of one sequence, by an explicit gather
    (independent of the oracle's paged walk)."""
    kd, ks, vd, vs = cache
    t = np.arange(n_tok)
    pages = page_table[seq, t // block_size]
    off = t % block_size

    def deq(d, s):
        b = d[pages, :, off, :]                        # [n_tok][Hkv][D/2] u8
        codes = np.stack([b & 15, b >> 4], -1).reshape(b.shape[0], b.shape[1], -1).astype(np.float64)
        sc = s[pages, :, off, :].view(np.float16).astype(np.float64)   # [n_tok][Hkv][D/32]
        return (codes - 8) * np.repeat(sc, 32, axis=-1)
    return deq(kd, ks), deq(vd, vs)


# ---------------------------------------------------------------------------
# device-side helpers for the GPU parity tests

def to_dev(a, device="cuda"):
    """numpy -> torch CUDA tensor; uint16 (bf16/fp16 bits) travel as int16."""
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def to_host(t, dtype=None):
    a = t.detach().cpu().numpy()
    if dtype is not None:
        a = a.view(dtype)
    return a


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (float64 in, float64 out)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


# The attention tolerance: 2e-3 on top of the bf16 rounding of the output
# (half a bf16 ulp of the exact value).
ATOL_ATTN = 2e-3


def attn_within(gpu_bf16_bits, ref_f64, atol=ATOL_ATTN):
    g = workloads.bf16_bits_to_f32(gpu_bf16_bits).astype(np.float64)
    err = np.abs(g - ref_f64)
    bound = atol + 0.5 * bf16_ulp(ref_f64)
    return err, bound


def split_bound(i, n, S, block, head_dim):
    """First page of split i of a sequence of n pages, as include/qkv.h states
    the plan: i * n / S, except that with S >= 8 the first ceil(S / 7) splits
    are d pages shorter (d = 400 tokens at head_dim 256, 800 at 128, at most a
    quarter split), the other splits sharing those pages."""
    m = (S + 6) // 7 if S >= 8 else 0
    d = min((400 if head_dim == 256 else 800) // block, n // S // 4)
    if m == 0 or d == 0:
        return i * n // S
    num = (i * n - i * d * S) * (S - m) if i <= m else n * (S - m) * i - m * d * S * (S - i)
    return num // (S * (S - m))
