"""Device memory plumbing around the C ABI: the paged F4 cache of one layer
and a decode-attention helper that owns its workspace. PyTorch supplies the
memory and streams; every computation is a library call."""
from __future__ import annotations

import dataclasses

import torch

from . import _abi


@dataclasses.dataclass
class PagedF4Cache:
    """One layer's F4 cache: data u8 [num_pages][kv_heads][block][head_dim/2]
    and fp16 scales [num_pages][kv_heads][block][head_dim/32], for K and V;
    with v_group=head_dim the V scales are [num_pages][kv_heads][block][1]
    (one per token and head). The library calls read the V layout from the
    last dimension of v_scale."""

    k_data: torch.Tensor
    k_scale: torch.Tensor
    v_data: torch.Tensor
    v_scale: torch.Tensor

    @classmethod
    def allocate(cls, num_pages: int, kv_heads: int, block_size: int, head_dim: int, device="cuda",
                 v_group: int = 32, pinned: bool = False):
        """pinned=True: a host-placed pool in page-locked host memory (device
        "cpu"), which the tier's kernels read in place over the host link."""
        if v_group not in (32, head_dim):
            raise ValueError(f"v_group must be 32 or head_dim ({head_dim}), got {v_group}")
        kw = dict(device="cpu", pin_memory=True) if pinned else dict(device=device)
        d = lambda: torch.zeros((num_pages, kv_heads, block_size, head_dim // 2), dtype=torch.uint8, **kw)
        s = lambda g: torch.zeros((num_pages, kv_heads, block_size, head_dim // g), dtype=torch.float16, **kw)
        return cls(d(), s(32), d(), s(v_group))

    @property
    def num_pages(self) -> int:
        return self.k_data.shape[0]

    @property
    def kv_heads(self) -> int:
        return self.k_data.shape[1]

    @property
    def block_size(self) -> int:
        return self.k_data.shape[2]

    @property
    def head_dim(self) -> int:
        return self.k_data.shape[3] * 2

    @property
    def v_group(self) -> int:
        return _abi.v_group_of(self.v_scale, self.head_dim)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.k_data, self.k_scale, self.v_data, self.v_scale))

    def write(self, k, v, slot_mapping, device_status=None, stream=None):
        _abi.qkv_kv_write_f4(k, v, slot_mapping, self.k_data, self.k_scale, self.v_data, self.v_scale,
                             device_status=device_status, stream=stream)


class DecodeAttention:
    """Split pass + log2-sum-exp merge with a workspace sized once."""

    def __init__(self, n_seq: int, q_heads: int, kv_heads: int, head_dim: int, block_size: int,
                 max_splits: int = 0, device="cuda"):
        self.kv_heads = kv_heads
        self.max_splits = max_splits or max(1, _abi.qkv_paged_decode_auto_splits(kv_heads, block_size))
        nbytes = _abi.qkv_paged_decode_workspace_bytes(n_seq, q_heads, head_dim, self.max_splits)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def partials(self, n_seq: int, q_heads: int, head_dim: int):
        """Views of the workspace as the split pass leaves it after a call:
        o_parts float [max_splits][n_seq * q_heads][head_dim] and lse2_parts
        float [max_splits][n_seq * q_heads] (-inf for a split slot that held
        no tokens), the layout include/qkv.h gives for the workspace."""
        rows = n_seq * q_heads * self.max_splits
        l0 = (rows * head_dim * 4 + 255) // 256 * 256
        o = self.workspace[:rows * head_dim * 4].view(torch.float32)
        lse = self.workspace[l0:l0 + rows * 4].view(torch.float32)
        return o.view(self.max_splits, n_seq * q_heads, head_dim), lse.view(self.max_splits, n_seq * q_heads)

    def step(self, out, q, k_new, v_new, positions, slot_mapping, cos_tab, sin_tab, table_pos_start: int,
             rot_dim: int, cache: PagedF4Cache, page_table, seq_lens, lse2_out=None, softmax_scale=0.0,
             num_splits=0, device_status=None, stream=None):
        """The layer's whole decode step (rotary, F4 write of the new token,
        attention, merge) in two launches; q unrotated."""
        _abi.qkv_decode_step_f4(out, q, k_new, v_new, positions, slot_mapping, cos_tab, sin_tab, table_pos_start,
                                rot_dim, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, page_table,
                                seq_lens, self.kv_heads, self.workspace, self.max_splits, lse2_out=lse2_out,
                                softmax_scale=softmax_scale, num_splits=num_splits, device_status=device_status,
                                stream=stream)

    def __call__(self, out, q, cache: PagedF4Cache, page_table, seq_lens, lse2_out=None, softmax_scale=0.0,
                 num_splits=0, device_status=None, stream=None):
        _abi.qkv_paged_decode_attn_f4(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                                      page_table, seq_lens, self.kv_heads, self.workspace, self.max_splits,
                                      lse2_out=lse2_out, softmax_scale=softmax_scale, num_splits=num_splits,
                                      device_status=device_status, stream=stream)


class TieredDecodeAttention:
    """Decode attention over a context split between a pinned host pool (the
    older tokens, whole pages) and the device pool, with the window and
    partials workspace sized once."""

    def __init__(self, q_heads: int, kv_heads: int, head_dim: int, block_size: int, max_host_pages_per_seq: int,
                 window_pages: int, v_group: int = 32, max_splits: int = 0, device="cuda"):
        self.kv_heads = kv_heads
        self.window_pages = window_pages
        self.max_splits = max_splits or max(1, _abi.qkv_paged_decode_auto_splits(kv_heads, block_size))
        nbytes = _abi.qkv_paged_decode_tiered_workspace_bytes(q_heads, kv_heads, head_dim, block_size, v_group,
                                                              max_host_pages_per_seq, window_pages, self.max_splits)
        if nbytes == 0:
            raise ValueError("invalid tiered-decode sizes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def __call__(self, out, q, cache: PagedF4Cache, page_table, seq_lens, host: PagedF4Cache, host_page_table,
                 host_lens, lse2_out=None, softmax_scale=0.0, device_status=None, stream=None):
        _abi.qkv_paged_decode_attn_f4_tiered(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                                             page_table, seq_lens, host.k_data, host.k_scale, host.v_data,
                                             host.v_scale, host_page_table, host_lens, self.kv_heads,
                                             self.window_pages, self.max_splits, self.workspace, lse2_out=lse2_out,
                                             softmax_scale=softmax_scale, device_status=device_status,
                                             stream=stream)


class TieredPrefillAttention:
    """Chunked prefill of one sequence whose oldest pages sit in a pinned host
    pool, with the window and partials workspace sized once."""

    def __init__(self, n_q: int, q_heads: int, kv_heads: int, head_dim: int, block_size: int, max_host_pages: int,
                 window_pages: int, v_group: int = 32, parts_per_launch: int = 4, device="cuda"):
        self.kv_heads = kv_heads
        self.window_pages = window_pages
        self.parts_per_launch = parts_per_launch
        nbytes = _abi.qkv_paged_prefill_tiered_workspace_bytes(n_q, q_heads, kv_heads, head_dim, block_size, v_group,
                                                               max_host_pages, window_pages, parts_per_launch)
        if nbytes == 0:
            raise ValueError("invalid tiered-prefill sizes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def __call__(self, out, q, cache: PagedF4Cache, page_table, prefix_len: int, host: PagedF4Cache,
                 host_page_table, host_len: int, lse2_out=None, softmax_scale=0.0, device_status=None, stream=None):
        _abi.qkv_paged_prefill_attn_f4_tiered(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                                              page_table, prefix_len, host.k_data, host.k_scale, host.v_data,
                                              host.v_scale, host_page_table, host_len, self.kv_heads,
                                              self.window_pages, self.parts_per_launch, self.workspace,
                                              lse2_out=lse2_out, softmax_scale=softmax_scale,
                                              device_status=device_status, stream=stream)
