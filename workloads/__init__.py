"""Seeded synthetic inputs for the decode hot path.

This module only draws random numbers and lays out page tables. It holds none
of the method's arithmetic (no rotary, no quantisation, no attention), so the
CPU oracle and the CUDA library can both consume its arrays without sharing
any code.

Two generators follow the same recipe:

* ``host``: numpy ``Generator(PCG64(seed))``; used for sizes the oracle handles
  in seconds.
* ``device``: torch's Philox generator on a CUDA device; used for the
  full-size workloads (hundreds of MB to GB per layer). Tests that need the
  oracle at full size copy these arrays to the host.

Values are N(0, 1) drawn in float64 (host) or float32 (device), optionally
multiplied by a per-head factor and an outlier factor, then rounded to float32
and from float32 to bfloat16 with round-to-nearest-even. Arrays are returned as
``uint16`` bit patterns (host) or ``torch.int16`` tensors holding the same bits
(device).

Workload shapes follow the serving pages: 16 query heads over 4 KV heads of
dimension 256, a 64-of-256 partial rotary, 64-token pages, contexts from 4,096
to 1,048,576 tokens.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

# Stream ids: each tensor of a layer draws from its own seeded stream.
STREAM_Q, STREAM_K_CACHE, STREAM_V_CACHE, STREAM_K_NEW, STREAM_V_NEW = 0, 1, 2, 3, 4
STREAM_HEAD_SCALE, STREAM_OUTLIER, STREAM_PAGES = 5, 6, 7
STREAM_CHUNK_Q = 8


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode-step workload.

    ``seq_lens`` counts every context token of a sequence, including the one
    the decode step writes: the cache is pre-filled with ``L - 1`` tokens at
    positions ``first_position ... first_position + L - 2`` and the step runs
    at position ``first_position + L - 1``. ``L = 0`` is an empty context:
    nothing is pre-filled, the step writes no token (its slot is -1) and its
    query is rotated at ``first_position``.
    """

    name: str
    n_layers: int
    seq_lens: Tuple[int, ...]
    num_pages: int
    block_size: int = 64
    q_heads: int = 16
    kv_heads: int = 4
    head_dim: int = 256
    rot_dim: int = 64
    rope_base: float = 1.0e7
    yarn_factor: float = 1.0
    orig_max_pos: int = 262144
    beta_fast: float = 32.0
    beta_slow: float = 1.0
    first_position: int = 0
    page_alloc: str = "contiguous"  # or "interleaved"
    head_scale: bool = False  # one U(0.5, 2) factor per head
    k_outlier_frac: float = 0.0  # share of (token, kv head) K vectors scaled
    k_outlier_mult: float = 20.0
    num_splits: int = 0  # 0: the library chooses
    seed: int = 0

    @property
    def n_seq(self) -> int:
        return len(self.seq_lens)

    @property
    def max_pages_per_seq(self) -> int:
        return max(-(-L // self.block_size) for L in self.seq_lens)

    @property
    def step_positions(self) -> List[int]:
        return [self.first_position + max(L - 1, 0) for L in self.seq_lens]

    def algorithmic_bytes_per_layer(self) -> int:
        """K/V data + fp16 scales of every context token, page-table entries,
        q in and bf16 out, for one layer's decode attention."""
        ctx = sum(self.seq_lens)
        d, hkv = self.head_dim, self.kv_heads
        kv = ctx * hkv * 2 * (d // 2 + (d // 32) * 2)
        pt = 4 * sum(-(-L // self.block_size) for L in self.seq_lens)
        qo = 2 * self.n_seq * self.q_heads * d * 2
        return kv + pt + qo


# The five serving workloads (names describe what they are).
TINY_4K = Workload(name="tiny_4k", n_layers=1, seq_lens=(4096,), num_pages=256, block_size=16,
                   num_splits=4)
CTX_131K = Workload(name="ctx131k_headscale", n_layers=16, seq_lens=(131072,), num_pages=2048,
                    head_scale=True)
YARN_262K = Workload(name="yarn262k", n_layers=16, seq_lens=(262144,), num_pages=4096,
                     yarn_factor=4.0, first_position=262144)
LANES_3 = Workload(name="lanes3_524k_pool", n_layers=16, seq_lens=(262144, 196608, 65536),
                   num_pages=8192, page_alloc="interleaved")
YARN_1M = Workload(name="yarn1m_outliers", n_layers=16, seq_lens=(1048576,), num_pages=16384,
                   yarn_factor=4.0, k_outlier_frac=0.01, num_splits=148)

ALL = (TINY_4K, CTX_131K, YARN_262K, LANES_3, YARN_1M)
BY_NAME = {w.name: w for w in ALL}


def small(name: str, seq_lens: Sequence[int], num_pages: int, block_size: int = 64, **kw) -> Workload:
    """A reduced workload with the same recipe, for oracle-sized tests."""
    return Workload(name=name, n_layers=1, seq_lens=tuple(seq_lens), num_pages=num_pages,
                    block_size=block_size, **kw)


# ---------------------------------------------------------------------------
# bit-level helpers (format conversion of generated values only)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit pattern, round to nearest even (finite input)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, layer: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, layer, stream]))


# ---------------------------------------------------------------------------
# page tables


def page_table(w: Workload) -> np.ndarray:
    """int32 [n_seq][max_pages_per_seq]; entries past a sequence's pages are -1.

    The physical pool is a seeded random permutation of ``num_pages`` pages.
    ``contiguous`` deals each sequence a contiguous run of the shuffled pool;
    ``interleaved`` deals pages round-robin to the sequences that still need
    pages, so neighbouring pages of the pool belong to different lanes.
    """
    need = [-(-L // w.block_size) for L in w.seq_lens]
    if sum(need) > w.num_pages:
        raise ValueError(f"{w.name}: {sum(need)} pages needed, pool has {w.num_pages}")
    perm = _rng(w.seed, 0, STREAM_PAGES).permutation(w.num_pages).astype(np.int32)
    pt = np.full((w.n_seq, w.max_pages_per_seq), -1, dtype=np.int32)
    if w.page_alloc == "contiguous":
        off = 0
        for s, n in enumerate(need):
            pt[s, :n] = perm[off:off + n]
            off += n
    elif w.page_alloc == "interleaved":
        filled = [0] * w.n_seq
        i = 0
        while any(filled[s] < need[s] for s in range(w.n_seq)):
            for s in range(w.n_seq):
                if filled[s] < need[s]:
                    pt[s, filled[s]] = perm[i]
                    filled[s] += 1
                    i += 1
    else:
        raise ValueError(w.page_alloc)
    return pt


def cache_slots(w: Workload, pt: np.ndarray) -> np.ndarray:
    """int64 slot (page * block_size + offset) of every pre-filled token, in
    the order of the generated K/V rows: sequence by sequence, token by token."""
    out = []
    for s, L in enumerate(w.seq_lens):
        t = np.arange(max(L - 1, 0), dtype=np.int64)
        out.append(pt[s, t // w.block_size].astype(np.int64) * w.block_size + t % w.block_size)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def step_slots(w: Workload, pt: np.ndarray) -> np.ndarray:
    """int64 slot of the token each sequence's decode step writes."""
    return np.array([int(pt[s, (L - 1) // w.block_size]) * w.block_size + (L - 1) % w.block_size if L > 0 else -1
                     for s, L in enumerate(w.seq_lens)], dtype=np.int64)


# ---------------------------------------------------------------------------
# host generator


def _head_factors(w: Workload, layer: int) -> Dict[str, np.ndarray]:
    if not w.head_scale:
        return {"q": np.ones(w.q_heads), "k": np.ones(w.kv_heads), "v": np.ones(w.kv_heads)}
    r = _rng(w.seed, layer, STREAM_HEAD_SCALE)
    return {"q": r.uniform(0.5, 2.0, w.q_heads), "k": r.uniform(0.5, 2.0, w.kv_heads),
            "v": r.uniform(0.5, 2.0, w.kv_heads)}


def head_factors(w: Workload, layer: int) -> Dict[str, np.ndarray]:
    """Per-head amplitude factors (all ones unless ``head_scale``)."""
    return _head_factors(w, layer)


def host_layer(w: Workload, layer: int = 0) -> Dict[str, np.ndarray]:
    """All inputs of one layer's decode step, as host arrays.

    Keys: ``q`` [n_seq][Hq][D], ``k_cache``/``v_cache`` [T][Hkv][D] (T = sum
    of max(L - 1, 0), rows ordered as ``cache_slots``), ``k_new``/``v_new``
    [n_seq][Hkv][D] (bf16 bits, uint16); ``page_table``, ``cache_slots``,
    ``step_slots``, ``seq_lens`` (int32), ``positions`` (int64, step position
    of each sequence).
    """
    f = _head_factors(w, layer)
    T = sum(max(L - 1, 0) for L in w.seq_lens)
    d = w.head_dim

    def normal(stream, shape, head_f, head_axis):
        x = _rng(w.seed, layer, stream).standard_normal(shape)
        bshape = [1] * len(shape)
        bshape[head_axis] = -1
        return x * head_f.reshape(bshape)

    q = normal(STREAM_Q, (w.n_seq, w.q_heads, d), f["q"], 1)
    kc = normal(STREAM_K_CACHE, (T, w.kv_heads, d), f["k"], 1)
    if w.k_outlier_frac > 0:
        m = _rng(w.seed, layer, STREAM_OUTLIER).random((T, w.kv_heads)) < w.k_outlier_frac
        kc = np.where(m[..., None], kc * w.k_outlier_mult, kc)
    vc = normal(STREAM_V_CACHE, (T, w.kv_heads, d), f["v"], 1)
    kn = normal(STREAM_K_NEW, (w.n_seq, w.kv_heads, d), f["k"], 1)
    vn = normal(STREAM_V_NEW, (w.n_seq, w.kv_heads, d), f["v"], 1)
    pt = page_table(w)
    to16 = lambda a: f32_to_bf16_bits(a.astype(np.float32))
    return {
        "q": to16(q), "k_cache": to16(kc), "v_cache": to16(vc), "k_new": to16(kn), "v_new": to16(vn),
        "page_table": pt, "cache_slots": cache_slots(w, pt), "step_slots": step_slots(w, pt),
        "seq_lens": np.array(w.seq_lens, dtype=np.int32),
        "positions": np.array(w.step_positions, dtype=np.int64),
    }


# ---------------------------------------------------------------------------
# device generator (torch Philox on CUDA); same recipe, different stream


def device_layer(w: Workload, layer: int, device) -> Dict[str, "object"]:
    """Same keys as ``host_layer``; bf16 arrays are ``torch.int16`` tensors on
    ``device`` holding bf16 bits, index arrays are device tensors too."""
    import torch

    f = _head_factors(w, layer)
    T = sum(max(L - 1, 0) for L in w.seq_lens)
    d = w.head_dim

    def gen(stream):
        g = torch.Generator(device=device)
        g.manual_seed((w.seed * 1_000_003 + layer) * 64 + stream)
        return g

    def normal(stream, shape, head_f):
        x = torch.randn(shape, generator=gen(stream), device=device, dtype=torch.float32)
        hf = torch.tensor(head_f, dtype=torch.float32, device=device).view(1, -1, 1)
        return x * hf

    def to16(x):
        return x.to(torch.bfloat16).view(torch.int16)

    q = to16(normal(STREAM_Q, (w.n_seq, w.q_heads, d), f["q"]))
    kc = normal(STREAM_K_CACHE, (T, w.kv_heads, d), f["k"])
    if w.k_outlier_frac > 0:
        m = torch.rand((T, w.kv_heads), generator=gen(STREAM_OUTLIER), device=device) < w.k_outlier_frac
        kc = torch.where(m.unsqueeze(-1), kc * w.k_outlier_mult, kc)
    kc = to16(kc)
    vc = to16(normal(STREAM_V_CACHE, (T, w.kv_heads, d), f["v"]))
    kn = to16(normal(STREAM_K_NEW, (w.n_seq, w.kv_heads, d), f["k"]))
    vn = to16(normal(STREAM_V_NEW, (w.n_seq, w.kv_heads, d), f["v"]))
    pt = page_table(w)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return {
        "q": q, "k_cache": kc, "v_cache": vc, "k_new": kn, "v_new": vn,
        "page_table": t(pt), "cache_slots": t(cache_slots(w, pt)), "step_slots": t(step_slots(w, pt)),
        "seq_lens": t(np.array(w.seq_lens, dtype=np.int32)),
        "positions": t(np.array(w.step_positions, dtype=np.int64)),
        "page_table_host": pt,
    }


def chunk_queries_host(w: Workload, layer: int, n_q: int) -> np.ndarray:
    """bf16 bits [n_q][Hq][D]: the queries of a prefill chunk (the last n_q
    tokens of the workload's single sequence), same value recipe as q."""
    f = _head_factors(w, layer)
    x = _rng(w.seed, layer, STREAM_CHUNK_Q).standard_normal((n_q, w.q_heads, w.head_dim))
    return f32_to_bf16_bits((x * f["q"].reshape(1, -1, 1)).astype(np.float32))


def chunk_queries_device(w: Workload, layer: int, n_q: int, device):
    """``chunk_queries_host`` drawn on the device (torch Philox)."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed((w.seed * 1_000_003 + layer) * 64 + STREAM_CHUNK_Q)
    x = torch.randn((n_q, w.q_heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    x = x * torch.tensor(_head_factors(w, layer)["q"], dtype=torch.float32, device=device).view(1, -1, 1)
    return x.to(torch.bfloat16).view(torch.int16)


def yarn_spec(w: Workload) -> Dict[str, float]:
    """The rotary configuration of a workload as plain numbers (no derived
    quantities: the ramp and attention factor are computed by each side)."""
    return {"rope_base": w.rope_base, "rot_dim": w.rot_dim, "factor": w.yarn_factor,
            "orig_max_pos": w.orig_max_pos, "beta_fast": w.beta_fast, "beta_slow": w.beta_slow}
