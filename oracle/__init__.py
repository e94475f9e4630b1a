"""fp64 CPU oracle of the decode hot path (ctypes front end of qkv_oracle.c).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library and
its Python binding never import it, and the two share no code: the only
common inputs are the arrays drawn by ``workloads``.

Every function takes and returns numpy arrays. bf16 and fp16 values travel as
``uint16`` bit patterns; results are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile qkv_oracle.c with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-D_DEFAULT_SOURCE", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib: Optional[ctypes.CDLL] = None


class YarnParams(ctypes.Structure):
    _fields_ = [("rope_base", ctypes.c_double), ("rot_dim", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("factor", ctypes.c_double), ("orig_max_pos", ctypes.c_int64),
                ("beta_fast", ctypes.c_double), ("beta_slow", ctypes.c_double),
                ("ext_factor", ctypes.c_double), ("attn_factor", ctypes.c_double)]


def _params(spec: Dict) -> YarnParams:
    return YarnParams(float(spec["rope_base"]), int(spec["rot_dim"]), 0, float(spec.get("factor", 1.0)),
                      int(spec.get("orig_max_pos", 262144)), float(spec.get("beta_fast", 32.0)),
                      float(spec.get("beta_slow", 1.0)), float(spec.get("ext_factor", -1.0)),
                      float(spec.get("attn_factor", 0.0)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        d, i32, i64, vp = ctypes.c_double, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
        P = ctypes.POINTER(YarnParams)
        sig = {
            "oracle_yarn_theta": (d, [P, vp, vp, vp]),
            "oracle_yarn_table": (None, [P, i64, i64, vp, vp]),
            "oracle_rope_apply_f64": (None, [vp, vp, vp, i32, i32, i32, P]),
            "oracle_rope_apply_bf16": (None, [vp, vp, vp, i32, i32, i32, P]),
            "oracle_quantize_cell": (None, [vp, vp, vp]),
            "oracle_quantize_group": (None, [vp, i32, vp, vp]),
            "oracle_kv_write_f4": (i32, [vp, vp, vp, i64, vp, vp, vp, vp, i32, i32, i32, i64, i32]),
            "oracle_paged_attention": (None, [vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i32,
                                              d, vp, vp, i32, i32]),
            "oracle_lse_merge": (None, [vp, vp, i32, i32, i32, vp, vp]),
            "oracle_gather_kv_f4": (i64, [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32, i64, i32, vp,
                                          vp]),
            "oracle_max_threads": (i32, []),
            "oracle_f64_to_f16_array": (None, [vp, vp, i64]),
            "oracle_f16_to_f64_array": (None, [vp, vp, i64]),
            "oracle_f64_to_bf16_array": (None, [vp, vp, i64]),
            "oracle_bf16_to_f64_array": (None, [vp, vp, i64]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype, fn.argtypes = res, args
    return _lib


def _p(a: np.ndarray) -> int:
    return a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# formats

def f64_to_f16(x) -> np.ndarray:
    x = _c(x, np.float64); y = np.empty(x.shape, np.uint16)
    lib().oracle_f64_to_f16_array(_p(x), _p(y), x.size); return y


def f16_to_f64(x) -> np.ndarray:
    x = _c(x, np.uint16); y = np.empty(x.shape, np.float64)
    lib().oracle_f16_to_f64_array(_p(x), _p(y), x.size); return y


def f64_to_bf16(x) -> np.ndarray:
    x = _c(x, np.float64); y = np.empty(x.shape, np.uint16)
    lib().oracle_f64_to_bf16_array(_p(x), _p(y), x.size); return y


def bf16_to_f64(x) -> np.ndarray:
    x = _c(x, np.uint16); y = np.empty(x.shape, np.float64)
    lib().oracle_bf16_to_f64_array(_p(x), _p(y), x.size); return y


# ---------------------------------------------------------------------------
# rotary

def yarn_theta(spec: Dict) -> Tuple[np.ndarray, float, float, float]:
    """(theta [rot_dim/2], mscale, low, high)."""
    p = _params(spec)
    th = np.empty(p.rot_dim // 2, np.float64)
    lo, hi = ctypes.c_double(), ctypes.c_double()
    ms = lib().oracle_yarn_theta(ctypes.byref(p), _p(th), ctypes.addressof(lo), ctypes.addressof(hi))
    return th, ms, lo.value, hi.value


def yarn_table(spec: Dict, pos0: int, n_pos: int) -> Tuple[np.ndarray, np.ndarray]:
    p = _params(spec)
    c = np.empty((n_pos, p.rot_dim // 2)); s = np.empty_like(c)
    lib().oracle_yarn_table(ctypes.byref(p), pos0, n_pos, _p(c), _p(s))
    return c, s


def rope_apply_f64(x, positions, spec: Dict) -> np.ndarray:
    """x float64 [n_tok][n_heads][head_dim] -> rotated copy (float64)."""
    x = _c(x, np.float64); pos = _c(positions, np.int64); y = np.empty_like(x)
    p = _params(spec)
    lib().oracle_rope_apply_f64(_p(x), _p(y), _p(pos), x.shape[0], x.shape[1], x.shape[2], ctypes.byref(p))
    return y


def rope_apply_bf16(x, positions, spec: Dict) -> np.ndarray:
    """x bf16 bits [n_tok][n_heads][head_dim] -> rotated bf16 bits."""
    x = _c(x, np.uint16); pos = _c(positions, np.int64); y = np.empty_like(x)
    p = _params(spec)
    lib().oracle_rope_apply_bf16(_p(x), _p(y), _p(pos), x.shape[0], x.shape[1], x.shape[2], ctypes.byref(p))
    return y


# ---------------------------------------------------------------------------
# F4 cache

def quantize_cell(x32) -> Tuple[np.ndarray, int]:
    x = _c(x32, np.uint16); assert x.size == 32
    b = np.empty(16, np.uint8); s = np.empty(1, np.uint16)
    lib().oracle_quantize_cell(_p(x), _p(b), _p(s))
    return b, int(s[0])


def quantize_group(x) -> Tuple[np.ndarray, int]:
    """One group of n values (n even) sharing a scale: (bytes [n/2], scale bits)."""
    x = _c(x, np.uint16); n = x.size; assert n % 2 == 0 and n <= 1024
    b = np.empty(n // 2, np.uint8); s = np.empty(1, np.uint16)
    lib().oracle_quantize_group(_p(x), n, _p(b), _p(s))
    return b, int(s[0])


def empty_cache(num_pages: int, kv_heads: int, block_size: int, head_dim: int, v_group: int = 32):
    """Zeroed (k_data, k_scale, v_data, v_scale) in the paged layout. K has
    one scale per 32-value cell; V one per v_group values (32, or head_dim for
    one scale per token, the PR's own V layout)."""
    data = lambda: np.zeros((num_pages, kv_heads, block_size, head_dim // 2), np.uint8)
    scale = lambda g: np.zeros((num_pages, kv_heads, block_size, head_dim // g), np.uint16)
    return data(), scale(32), data(), scale(v_group)


def v_group_of(cache, head_dim: int) -> int:
    """Values per V scale of a cache from empty_cache."""
    return head_dim // cache[3].shape[-1]


def kv_write_f4(k, v, slots, cache, kv_heads: int, head_dim: int, block_size: int) -> int:
    """Quantise rows of k, v (bf16 bits [n_tok][kv_heads][head_dim]) into
    ``cache`` (in place) at ``slots``; returns the number of bad slots."""
    k = _c(k, np.uint16); v = _c(v, np.uint16); sl = _c(slots, np.int64)
    kd, ks, vd, vs = cache
    for a in cache:
        assert a.flags.c_contiguous
    return lib().oracle_kv_write_f4(_p(k), _p(v), _p(sl), sl.size, _p(kd), _p(ks), _p(vd), _p(vs),
                                    kv_heads, head_dim, block_size, kd.shape[0], v_group_of(cache, head_dim))


# ---------------------------------------------------------------------------
# attention

def paged_attention(q, cache, page_table, tok_begin, tok_end, q_heads: int, kv_heads: int,
                    head_dim: int, block_size: int, softmax_scale: Optional[float] = None,
                    n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention per (sequence, query head) over the token range
    [tok_begin[s], tok_end[s]). Returns (out [n_seq][Hq][D], lse2 [n_seq][Hq])."""
    q = _c(q, np.uint16); pt = _c(page_table, np.int32)
    tb = _c(tok_begin, np.int32); te = _c(tok_end, np.int32)
    n_seq = pt.shape[0]
    kd, ks, vd, vs = (np.ascontiguousarray(a) for a in cache)
    out = np.empty((n_seq, q_heads, head_dim)); lse2 = np.empty((n_seq, q_heads))
    sc = float(softmax_scale) if softmax_scale else 1.0 / np.sqrt(head_dim)
    lib().oracle_paged_attention(_p(q), _p(kd), _p(ks), _p(vd), _p(vs), _p(pt), pt.shape[1], _p(tb), _p(te),
                                 n_seq, q_heads, kv_heads, head_dim, block_size, sc, _p(out), _p(lse2),
                                 n_threads, v_group_of(cache, head_dim))
    return out, lse2


def gather_kv_f4(cache, page_table, seq_lens, out_start, kv_heads: int, head_dim: int, block_size: int,
                 n_out: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray, int]:
    """Dequantise each sequence's context tokens into contiguous rows:
    (k_out, v_out) bf16 bits [n_out][kv_heads][head_dim], sequence s at rows
    out_start[s] .. out_start[s] + seq_lens[s] - 1; plus the number of tokens
    whose page id was outside the pool (their rows are zero)."""
    pt = _c(page_table, np.int32); sl = _c(seq_lens, np.int32); st = _c(out_start, np.int64)
    kd, ks, vd, vs = (np.ascontiguousarray(a) for a in cache)
    if n_out is None:
        n_out = int(np.max(st + sl, initial=0))
    k_out = np.zeros((n_out, kv_heads, head_dim), np.uint16); v_out = np.zeros_like(k_out)
    bad = lib().oracle_gather_kv_f4(_p(kd), _p(ks), _p(vd), _p(vs), _p(pt), pt.shape[1], _p(sl), _p(st),
                                    pt.shape[0], kv_heads, head_dim, block_size, kd.shape[0],
                                    v_group_of(cache, head_dim), _p(k_out), _p(v_out))
    return k_out, v_out, int(bad)


def prefill_attention(q, cache, page_table_row, positions, q_heads: int, kv_heads: int, head_dim: int,
                      block_size: int, softmax_scale: Optional[float] = None,
                      n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Causal attention of a chunk of queries of one sequence against its
    paged cache [CHUNK]: query i (at position positions[i]) attends the
    cached tokens 0 .. positions[i]. That is paged_attention with one
    single-query "sequence" per chunk row, all on the same page-table row.
    Returns (out [n][Hq][D], lse2 [n][Hq])."""
    pos = _c(positions, np.int64)
    n = pos.size
    row = _c(page_table_row, np.int32).reshape(1, -1)
    pt = np.repeat(row, n, axis=0)
    return paged_attention(q, cache, pt, np.zeros(n, np.int32), (pos + 1).astype(np.int32), q_heads, kv_heads,
                           head_dim, block_size, softmax_scale, n_threads)


def tiered_attention(q, host_cache, host_page_table, host_lens, dev_cache, dev_page_table, dev_lens,
                     q_heads: int, kv_heads: int, head_dim: int, block_size: int,
                     softmax_scale: Optional[float] = None, n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Exact decode attention over a context held in two pools [TIER]
    (FreeToken issue #568, proposed solution item 2: the K/V of a long
    context kept in host RAM beside the device's pages). The context of
    sequence s is host_lens[s] tokens walked through host_page_table[s] in
    the host pool, then dev_lens[s] tokens walked through dev_page_table[s] in
    the device pool. host_lens are whole pages. Written as paged_attention
    over one pool holding both (device page ids shifted past the host pool's
    pages) and one page-table row per sequence: host pages, then device pages.
    Returns (out [n_seq][Hq][D], lse2 [n_seq][Hq])."""
    hl = np.asarray(host_lens, np.int64); dl = np.asarray(dev_lens, np.int64)
    hpt = np.asarray(host_page_table, np.int64); dpt = np.asarray(dev_page_table, np.int64)
    if np.any(hl % block_size):
        raise ValueError("host_lens must be whole pages")
    n_host_pages = host_cache[0].shape[0]
    pool = tuple(np.concatenate([np.ascontiguousarray(h), np.ascontiguousarray(d)]) for h, d in
                 zip(host_cache, dev_cache))
    n_seq = hl.size
    width = hpt.shape[1] + dpt.shape[1]
    pt = np.zeros((n_seq, width), np.int32)
    for s in range(n_seq):
        nh = int(hl[s]) // block_size
        nd = -(-int(dl[s]) // block_size)
        pt[s, :nh] = hpt[s, :nh]
        pt[s, nh:nh + nd] = dpt[s, :nd] + n_host_pages
    return paged_attention(q, pool, pt, np.zeros(n_seq, np.int32), (hl + dl).astype(np.int32), q_heads, kv_heads,
                           head_dim, block_size, softmax_scale, n_threads)


def _two_pool_row(host_cache, host_row, host_len: int, dev_cache, dev_row, dev_tokens: int, block_size: int):
    """One pool holding both (device page ids shifted past the host pool's
    pages) and the page-table row: host pages, then device pages."""
    if host_len % block_size:
        raise ValueError("host_len must be whole pages")
    pool = tuple(np.concatenate([np.ascontiguousarray(h), np.ascontiguousarray(d)]) for h, d in
                 zip(host_cache, dev_cache))
    nh, nd = host_len // block_size, -(-dev_tokens // block_size)
    row = np.zeros(max(1, nh + nd), np.int32)
    row[:nh] = np.asarray(host_row, np.int64)[:nh]
    row[nh:nh + nd] = np.asarray(dev_row, np.int64)[:nd] + host_cache[0].shape[0]
    return pool, row


def tiered_prefill_attention(q, host_cache, host_row, host_len: int, dev_cache, dev_row, positions, q_heads: int,
                             kv_heads: int, head_dim: int, block_size: int, softmax_scale: Optional[float] = None,
                             n_threads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Causal attention of a chunk of queries of one sequence whose first
    host_len tokens (whole pages, row host_row) sit in the host pool [TIER]
    (FreeToken issue #568, proposed solution item 2: a prefill over host-placed
    K/V). Query i sits at device token positions[i] of dev_row and attends
    all host tokens and device tokens 0 .. positions[i]: prefill_attention
    over the sequence's whole context (host tokens first) at position
    host_len + positions[i]. Returns (out [n][Hq][D], lse2 [n][Hq])."""
    pos = np.asarray(positions, np.int64)
    pool, row = _two_pool_row(host_cache, host_row, host_len, dev_cache, dev_row, int(pos.max(initial=-1)) + 1,
                              block_size)
    return prefill_attention(q, pool, row, host_len + pos, q_heads, kv_heads, head_dim, block_size, softmax_scale,
                             n_threads)


def lse_merge(o_parts, lse2_parts) -> Tuple[np.ndarray, np.ndarray]:
    """o_parts [n_parts][rows][D], lse2_parts [n_parts][rows] -> (out, lse2)."""
    o = _c(o_parts, np.float64); l = _c(lse2_parts, np.float64)
    n, rows, d = o.shape
    out = np.empty((rows, d)); lse2 = np.empty(rows)
    lib().oracle_lse_merge(_p(o), _p(l), n, rows, d, _p(out), _p(lse2))
    return out, lse2


def max_threads() -> int:
    return lib().oracle_max_threads()


def dense_attention(q, k, v, softmax_scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of one sequence over unquantised K/V: the plain
    definition out = softmax(q k^T * scale) v, in float64 (the bf16 "oracle
    format" the ignis docs "context-and-speculation" run every correctness
    check against, KV pool section, --model-kv-format).

    q bf16 bits [Hq][D]; k, v bf16 bits [T][Hkv][D] (or float arrays); query
    head h reads KV head h // (Hq / Hkv). Returns (out [Hq][D], lse2 [Hq]),
    lse2 = log2 sum_t exp(score_t)."""
    def f64(a):
        a = np.asarray(a)
        return bf16_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)
    qf, kf, vf = f64(q), f64(k), f64(v)
    hq, d = qf.shape
    hkv = kf.shape[1]
    g = hq // hkv
    sc = float(softmax_scale) if softmax_scale else 1.0 / np.sqrt(d)
    out = np.zeros((hq, d))
    lse2 = np.full(hq, -np.inf)
    if kf.shape[0] == 0:
        return out, lse2
    for h in range(hq):
        s = kf[:, h // g, :] @ qf[h] * sc                    # [T]
        m = s.max()
        e = np.exp(s - m)
        z = e.sum()
        out[h] = (e @ vf[:, h // g, :]) / z
        lse2[h] = (m + np.log(z)) / np.log(2.0)
    return out, lse2
