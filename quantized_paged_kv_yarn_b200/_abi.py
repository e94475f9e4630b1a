"""ctypes declarations of include/qkv.h and argument marshalling."""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqkv.so")

QKV_OK, QKV_EINVAL, QKV_EUNSUPPORTED, QKV_ECUDA = 0, 1, 2, 3
DEV_BAD_POSITION, DEV_BAD_SLOT, DEV_BAD_PAGE, DEV_BAD_SEQLEN, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10


class QkvError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {qkv_status_string(code)} (status {code})")
        self.code = code


class YarnParams(ctypes.Structure):
    """Mirror of qkv_yarn_params."""
    _fields_ = [("rope_base", ctypes.c_double), ("rot_dim", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("factor", ctypes.c_double), ("orig_max_pos", ctypes.c_int64),
                ("beta_fast", ctypes.c_double), ("beta_slow", ctypes.c_double),
                ("ext_factor", ctypes.c_double), ("attn_factor", ctypes.c_double)]

    @classmethod
    def make(cls, rope_base=1e7, rot_dim=64, factor=1.0, orig_max_pos=262144, beta_fast=32.0, beta_slow=1.0,
             ext_factor=-1.0, attn_factor=0.0):
        return cls(float(rope_base), int(rot_dim), 0, float(factor), int(orig_max_pos), float(beta_fast),
                   float(beta_slow), float(ext_factor), float(attn_factor))


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python quantized_paged_kv_yarn_b200/build.py`")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i32, _i64, _f32, _f64, _sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                    ctypes.c_double, ctypes.c_size_t)
_SIGS = {
    "qkv_yarn_auto_factor": (_f64, [_i64, _i64]),
    "qkv_yarn_rope_table": (ctypes.c_int, [ctypes.POINTER(YarnParams), _i64, _i64, _vp, _vp, _vp]),
    "qkv_rope_apply": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i64, _i64, _vp, _vp]),
    "qkv_kv_write_f4": (ctypes.c_int, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i64, _vp,
                                       _vp]),
    "qkv_rope_kv_write_f4": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp,
                                            _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i64, _vp, _vp]),
    "qkv_paged_decode_auto_splits": (_i32, [_i32, _i32]),
    "qkv_paged_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "qkv_paged_decode_split_f4": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                                 _i32, _i32, _i32, _i32, _i64, _f32, _i32, _vp, _vp]),
    "qkv_lse_merge": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "qkv_paged_decode_attn_f4": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                _i32, _i32, _i32, _i64, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    "qkv_paged_decode_attn_f4_static": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                                       _i32, _i32, _i32, _i32, _i64, _f32, _i32, _vp, _vp]),
    "qkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qkv_kv_write_f4_v": (ctypes.c_int, [_vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i64, _i32, _vp,
                                         _vp]),
    "qkv_rope_kv_write_f4_v": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                              _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _i64, _i32, _vp, _vp]),
    "qkv_paged_decode_split_f4_v": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32,
                                                   _i32, _i32, _i32, _i32, _i64, _f32, _i32, _i32, _vp, _vp]),
    "qkv_paged_decode_attn_f4_v": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                  _i32, _i32, _i32, _i64, _f32, _i32, _i32, _i32, _vp, _sz, _vp,
                                                  _vp]),
    "qkv_gather_kv_f4": (ctypes.c_int, [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                        _i32, _i64, _i32, _vp, _vp]),
    "qkv_paged_prefill_attn_f4": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                                 _i32, _i32, _i32, _i64, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    "qkv_paged_prefill_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "qkv_decode_step_f4": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i64, _f32, _i32,
                                          _i32, _i32, _vp, _sz, _vp, _vp]),
    "qkv_decode_step_split_f4": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32,
                                                _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i64,
                                                _f32, _i32, _i32, _vp, _vp]),
    "qkv_stage_pages_f4": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _i32,
                                          _i32, _i32, _i32, _vp, _vp]),
    "qkv_paged_decode_tiered_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "qkv_paged_decode_attn_f4_tiered": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i64, _vp,
                                                       _vp, _vp, _vp, _i64, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                                       _i32, _i32, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
    "qkv_paged_prefill_auto_splits": (_i32, [_i32, _i32, _i32, _i32, _i32, _sz]),
    "qkv_paged_prefill_tiered_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "qkv_paged_prefill_attn_f4_tiered": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                        _i64, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _i32,
                                                        _i32, _i32, _f32, _i32, _i32, _vp, _sz, _vp, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype, _fn.argtypes = _res, _args


def exported_symbols():
    return sorted(_SIGS)


def qkv_status_string(code: int) -> str:
    return lib.qkv_status_string(int(code)).decode()


def _check(fn: str, rc: int):
    if rc != QKV_OK:
        raise QkvError(fn, rc)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


_U16 = (torch.bfloat16, torch.float16, torch.int16, torch.uint16)


def _ptr(t: Optional[torch.Tensor], name: str, dtypes=None, numel=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: has {t.numel()} elements, needs {numel}")
    return t.data_ptr()


def qkv_yarn_auto_factor(max_context: int, orig_max_pos: int = 262144) -> float:
    return lib.qkv_yarn_auto_factor(int(max_context), int(orig_max_pos))


def qkv_yarn_rope_table(params: YarnParams, pos_start: int, n_pos: int, cos_out: torch.Tensor,
                        sin_out: torch.Tensor, stream=None):
    n = n_pos * (params.rot_dim // 2)
    _check("qkv_yarn_rope_table", lib.qkv_yarn_rope_table(
        ctypes.byref(params), int(pos_start), int(n_pos), _ptr(cos_out, "cos_out", (torch.float32,), n),
        _ptr(sin_out, "sin_out", (torch.float32,), n), _stream(stream)))


def qkv_rope_apply(x_in, x_out, positions, cos_tab, sin_tab, table_pos_start: int, rot_dim: int,
                   device_status=None, stream=None):
    """x_in/x_out bf16 [n_tok][n_heads][head_dim] (x_out may be x_in)."""
    n_tok, n_heads, head_dim = x_in.shape
    if tuple(x_out.shape) != (n_tok, n_heads, head_dim):
        raise ValueError("x_out shape")
    half = rot_dim // 2
    _check("qkv_rope_apply", lib.qkv_rope_apply(
        _ptr(x_in, "x_in", _U16), _ptr(x_out, "x_out", _U16), _ptr(positions, "positions", (torch.int64,), n_tok),
        n_tok, n_heads, head_dim, rot_dim, _ptr(cos_tab, "cos_tab", (torch.float32,)),
        _ptr(sin_tab, "sin_tab", (torch.float32,)), int(table_pos_start), cos_tab.numel() // half,
        _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def v_group_of(v_scale, head_dim: int) -> int:
    """Values per V scale of a cache: 32 (per cell) or head_dim (per token)."""
    return head_dim // v_scale.shape[-1]


def qkv_kv_write_f4(k, v, slot_mapping, k_data, k_scale, v_data, v_scale, device_status=None, stream=None):
    """k/v bf16 [n_tok][kv_heads][head_dim]; cache tensors shaped
    [num_pages][kv_heads][block_size][head_dim/2 | head_dim/32]; v_scale's
    last dim 1 selects one V scale per token (qkv_kv_write_f4_v)."""
    n_tok, kv_heads, head_dim = k.shape
    num_pages, kvh2, block_size, half_bytes = k_data.shape
    if kvh2 != kv_heads or half_bytes != head_dim // 2 or tuple(v.shape) != tuple(k.shape):
        raise ValueError("cache/input shapes disagree")
    if slot_mapping.numel() != n_tok:
        raise ValueError(f"slot_mapping has {slot_mapping.numel()} entries for {n_tok} tokens")
    args = (_ptr(k, "k", _U16), _ptr(v, "v", _U16), _ptr(slot_mapping, "slot_mapping", (torch.int64,), n_tok), n_tok,
            _ptr(k_data, "k_data", (torch.uint8,)), _ptr(k_scale, "k_scale", _U16),
            _ptr(v_data, "v_data", (torch.uint8,)), _ptr(v_scale, "v_scale", _U16), kv_heads, head_dim, block_size,
            num_pages)
    tail = (_ptr(device_status, "device_status", (torch.int32,)), _stream(stream))
    vg = v_group_of(v_scale, head_dim)
    if vg == 32:
        _check("qkv_kv_write_f4", lib.qkv_kv_write_f4(*args, *tail))
    else:
        _check("qkv_kv_write_f4_v", lib.qkv_kv_write_f4_v(*args, vg, *tail))


def qkv_rope_kv_write_f4(q_in, q_out, k_in, v_in, positions, slot_mapping, cos_tab, sin_tab, table_pos_start: int,
                         rot_dim: int, k_data, k_scale, v_data, v_scale, k_out=None, device_status=None, stream=None):
    """Rotary of q (q_in -> q_out) and of k, and the F4 write of the rotated k
    and of v, in one launch."""
    n_tok, q_heads, head_dim = q_in.shape
    _, kv_heads, _ = k_in.shape
    num_pages, _, block_size, _ = k_data.shape
    half = rot_dim // 2
    if (tuple(q_out.shape) != tuple(q_in.shape) or tuple(k_in.shape) != (n_tok, kv_heads, head_dim)
            or tuple(v_in.shape) != tuple(k_in.shape) or (k_out is not None and tuple(k_out.shape) != tuple(k_in.shape))):
        raise ValueError("q/k/v shapes disagree")
    if slot_mapping.numel() != n_tok or positions.numel() != n_tok:
        raise ValueError("positions and slot_mapping need one entry per token")
    args = (_ptr(q_in, "q_in", _U16), _ptr(q_out, "q_out", _U16), _ptr(k_in, "k_in", _U16), _ptr(v_in, "v_in", _U16),
            _ptr(k_out, "k_out", _U16), _ptr(positions, "positions", (torch.int64,), n_tok),
            _ptr(slot_mapping, "slot_mapping", (torch.int64,), n_tok), n_tok, q_heads, kv_heads, head_dim, rot_dim,
            _ptr(cos_tab, "cos_tab", (torch.float32,)), _ptr(sin_tab, "sin_tab", (torch.float32,)),
            int(table_pos_start), cos_tab.numel() // half, *_cache_args(k_data, k_scale, v_data, v_scale), block_size,
            num_pages)
    tail = (_ptr(device_status, "device_status", (torch.int32,)), _stream(stream))
    vg = v_group_of(v_scale, head_dim)
    if vg == 32:
        _check("qkv_rope_kv_write_f4", lib.qkv_rope_kv_write_f4(*args, *tail))
    else:
        _check("qkv_rope_kv_write_f4_v", lib.qkv_rope_kv_write_f4_v(*args, vg, *tail))


def qkv_paged_decode_auto_splits(kv_heads: int, block_size: int) -> int:
    return lib.qkv_paged_decode_auto_splits(int(kv_heads), int(block_size))


def qkv_paged_decode_workspace_bytes(n_seq: int, q_heads: int, head_dim: int, max_splits: int) -> int:
    return lib.qkv_paged_decode_workspace_bytes(int(n_seq), int(q_heads), int(head_dim), int(max_splits))


def _cache_args(k_data, k_scale, v_data, v_scale):
    return (_ptr(k_data, "k_data", (torch.uint8,)), _ptr(k_scale, "k_scale", _U16),
            _ptr(v_data, "v_data", (torch.uint8,)), _ptr(v_scale, "v_scale", _U16))


def qkv_paged_decode_split_f4(o_parts, lse2_parts, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens,
                              kv_heads: int, softmax_scale: float = 0.0, num_splits: int = 0,
                              device_status=None, stream=None):
    """o_parts float [max_splits][n_seq*q_heads][head_dim], lse2_parts float
    [max_splits][n_seq*q_heads]."""
    n_seq, q_heads, head_dim = q.shape
    max_splits = o_parts.shape[0]
    num_pages, _, block_size, _ = k_data.shape
    args = (_ptr(o_parts, "o_parts", (torch.float32,), max_splits * n_seq * q_heads * head_dim),
            _ptr(lse2_parts, "lse2_parts", (torch.float32,), max_splits * n_seq * q_heads), max_splits,
            _ptr(q, "q", _U16), *_cache_args(k_data, k_scale, v_data, v_scale),
            _ptr(page_table, "page_table", (torch.int32,)), _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq),
            n_seq, q_heads, kv_heads, head_dim, block_size, page_table.shape[1], num_pages, float(softmax_scale),
            int(num_splits))
    tail = (_ptr(device_status, "device_status", (torch.int32,)), _stream(stream))
    vg = v_group_of(v_scale, head_dim)
    if vg == 32:
        _check("qkv_paged_decode_split_f4", lib.qkv_paged_decode_split_f4(*args, *tail))
    else:
        _check("qkv_paged_decode_split_f4_v", lib.qkv_paged_decode_split_f4_v(*args, vg, *tail))


def qkv_lse_merge(o_parts, lse2_parts, out, lse2_out=None, stream=None):
    """o_parts float [n_parts][rows][head_dim] -> out bf16 [rows][head_dim]."""
    n_parts, rows, head_dim = o_parts.shape
    _check("qkv_lse_merge", lib.qkv_lse_merge(
        _ptr(o_parts, "o_parts", (torch.float32,)), _ptr(lse2_parts, "lse2_parts", (torch.float32,), n_parts * rows),
        n_parts, rows, head_dim, _ptr(out, "out", _U16, rows * head_dim),
        _ptr(lse2_out, "lse2_out", (torch.float32,), rows), _stream(stream)))


def qkv_paged_decode_attn_f4(out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, kv_heads: int,
                             workspace, max_splits: int, lse2_out=None, softmax_scale: float = 0.0,
                             num_splits: int = 0, device_status=None, stream=None):
    """out bf16 [n_seq][q_heads][head_dim]; workspace a uint8 CUDA tensor of
    at least qkv_paged_decode_workspace_bytes(...) bytes."""
    n_seq, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    args = (_ptr(out, "out", _U16, n_seq * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,)),
            _ptr(q, "q", _U16), *_cache_args(k_data, k_scale, v_data, v_scale),
            _ptr(page_table, "page_table", (torch.int32,)), _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq),
            n_seq, q_heads, kv_heads, head_dim, block_size, page_table.shape[1], num_pages, float(softmax_scale),
            int(num_splits), int(max_splits))
    ws = (_ptr(workspace, "workspace"), workspace.numel() * workspace.element_size())
    tail = (_ptr(device_status, "device_status", (torch.int32,)), _stream(stream))
    vg = v_group_of(v_scale, head_dim)
    if vg == 32:
        _check("qkv_paged_decode_attn_f4", lib.qkv_paged_decode_attn_f4(*args, *ws, *tail))
    else:
        _check("qkv_paged_decode_attn_f4_v", lib.qkv_paged_decode_attn_f4_v(*args, vg, *ws, *tail))


def qkv_gather_kv_f4(k_out, v_out, k_data, k_scale, v_data, v_scale, page_table, seq_lens, out_start,
                     device_status=None, stream=None):
    """k_out/v_out bf16 [n_out][kv_heads][head_dim]; out_start int64 [n_seq]."""
    num_pages, kv_heads, block_size, half = k_data.shape
    head_dim = 2 * half
    n_seq = seq_lens.numel()
    if k_out.shape[1:] != (kv_heads, head_dim) or v_out.shape != k_out.shape:
        raise ValueError("k_out and v_out must be [n_out][kv_heads][head_dim]")
    _check("qkv_gather_kv_f4", lib.qkv_gather_kv_f4(
        _ptr(k_out, "k_out", _U16), _ptr(v_out, "v_out", _U16), k_out.shape[0],
        *_cache_args(k_data, k_scale, v_data, v_scale), _ptr(page_table, "page_table", (torch.int32,)),
        _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq), _ptr(out_start, "out_start", (torch.int64,), n_seq),
        n_seq, kv_heads, head_dim, block_size, page_table.shape[1], num_pages, v_group_of(v_scale, head_dim),
        _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def qkv_paged_prefill_workspace_bytes(n_q: int, q_heads: int, head_dim: int, num_splits: int) -> int:
    return lib.qkv_paged_prefill_workspace_bytes(int(n_q), int(q_heads), int(head_dim), int(num_splits))


def qkv_paged_prefill_attn_f4(out, q, k_data, k_scale, v_data, v_scale, page_table, prefix_len: int,
                              kv_heads: int, lse2_out=None, softmax_scale: float = 0.0, num_splits: int = 0,
                              workspace=None, device_status=None, stream=None):
    """out, q bf16 [n_q][q_heads][head_dim]; page_table int32 [max_pages] (one
    sequence); the chunk's queries sit at cache tokens prefix_len .. prefix_len + n_q - 1.
    workspace: a uint8 CUDA tensor (qkv_paged_prefill_workspace_bytes) or None."""
    n_q, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    page_table = page_table.reshape(-1)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("qkv_paged_prefill_attn_f4", lib.qkv_paged_prefill_attn_f4(
        _ptr(out, "out", _U16, n_q * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,), n_q * q_heads),
        _ptr(q, "q", _U16), *_cache_args(k_data, k_scale, v_data, v_scale),
        _ptr(page_table, "page_table", (torch.int32,)), n_q, int(prefix_len), q_heads, kv_heads, head_dim,
        block_size, page_table.numel(), num_pages, float(softmax_scale), v_group_of(v_scale, head_dim),
        int(num_splits), _ptr(workspace, "workspace"), ws_bytes, _ptr(device_status, "device_status", (torch.int32,)),
        _stream(stream)))


def qkv_decode_step_f4(out, q, k_new, v_new, positions, slot_mapping, cos_tab, sin_tab, table_pos_start: int,
                       rot_dim: int, k_data, k_scale, v_data, v_scale, page_table, seq_lens, kv_heads: int, workspace,
                       max_splits: int, lse2_out=None, softmax_scale: float = 0.0, num_splits: int = 0,
                       device_status=None, stream=None):
    """One layer's decode step (rotary, F4 write of the new k/v, attention,
    merge) in two launches; q unrotated. Shapes as in qkv_rope_kv_write_f4
    and qkv_paged_decode_attn_f4."""
    n_seq, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    half = rot_dim // 2
    _check("qkv_decode_step_f4", lib.qkv_decode_step_f4(
        _ptr(out, "out", _U16, n_seq * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,)),
        _ptr(q, "q", _U16), _ptr(k_new, "k_new", _U16, n_seq * kv_heads * head_dim),
        _ptr(v_new, "v_new", _U16, n_seq * kv_heads * head_dim), _ptr(positions, "positions", (torch.int64,), n_seq),
        _ptr(slot_mapping, "slot_mapping", (torch.int64,), n_seq), _ptr(cos_tab, "cos_tab", (torch.float32,)),
        _ptr(sin_tab, "sin_tab", (torch.float32,)), int(table_pos_start), cos_tab.numel() // half, int(rot_dim),
        *_cache_args(k_data, k_scale, v_data, v_scale), _ptr(page_table, "page_table", (torch.int32,)),
        _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq), n_seq, q_heads, kv_heads, head_dim, block_size,
        page_table.shape[1], num_pages, float(softmax_scale), int(num_splits), int(max_splits),
        v_group_of(v_scale, head_dim), _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def qkv_decode_step_split_f4(o_parts, lse2_parts, q, k_new, v_new, positions, slot_mapping, cos_tab, sin_tab,
                             table_pos_start: int, rot_dim: int, k_data, k_scale, v_data, v_scale, page_table,
                             seq_lens, kv_heads: int, softmax_scale: float = 0.0, num_splits: int = 0,
                             device_status=None, stream=None):
    """The decode step's split pass alone (rotary, F4 write of the new k/v,
    partials); o_parts / lse2_parts as in qkv_paged_decode_split_f4."""
    n_seq, q_heads, head_dim = q.shape
    max_splits = o_parts.shape[0]
    num_pages, _, block_size, _ = k_data.shape
    half = rot_dim // 2
    _check("qkv_decode_step_split_f4", lib.qkv_decode_step_split_f4(
        _ptr(o_parts, "o_parts", (torch.float32,), max_splits * n_seq * q_heads * head_dim),
        _ptr(lse2_parts, "lse2_parts", (torch.float32,), max_splits * n_seq * q_heads), max_splits,
        _ptr(q, "q", _U16), _ptr(k_new, "k_new", _U16, n_seq * kv_heads * head_dim),
        _ptr(v_new, "v_new", _U16, n_seq * kv_heads * head_dim), _ptr(positions, "positions", (torch.int64,), n_seq),
        _ptr(slot_mapping, "slot_mapping", (torch.int64,), n_seq), _ptr(cos_tab, "cos_tab", (torch.float32,)),
        _ptr(sin_tab, "sin_tab", (torch.float32,)), int(table_pos_start), cos_tab.numel() // half, int(rot_dim),
        *_cache_args(k_data, k_scale, v_data, v_scale), _ptr(page_table, "page_table", (torch.int32,)),
        _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq), n_seq, q_heads, kv_heads, head_dim, block_size,
        page_table.shape[1], num_pages, float(softmax_scale), int(num_splits), v_group_of(v_scale, head_dim),
        _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


STATIC_SCRATCH_BYTES = 16 << 20


def qkv_paged_decode_attn_f4_static(out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, kv_heads: int,
                                    lse2_out=None, softmax_scale: float = 0.0, num_splits: int = 0,
                                    device_status=None, stream=None):
    """Decode attention with the partials in the library's own device array
    (no workspace argument, no allocation). For callers that cannot allocate
    device memory; see include/qkv.h for the size limit and the rule that
    overlapping calls race on the shared array."""
    n_seq, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    if v_group_of(v_scale, head_dim) != 32:
        raise ValueError("qkv_paged_decode_attn_f4_static takes caches with one V scale per 32-value cell")
    _check("qkv_paged_decode_attn_f4_static", lib.qkv_paged_decode_attn_f4_static(
        _ptr(out, "out", _U16, n_seq * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,)),
        _ptr(q, "q", _U16), *_cache_args(k_data, k_scale, v_data, v_scale),
        _ptr(page_table, "page_table", (torch.int32,)), _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq), n_seq,
        q_heads, kv_heads, head_dim, block_size, page_table.shape[1], num_pages, float(softmax_scale),
        int(num_splits), _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def _hptr(t: torch.Tensor, name: str, dtypes=None, numel=None):
    """A device tensor, or a pinned (page-locked) host tensor that kernels
    read in place over the host link."""
    if isinstance(t, torch.Tensor) and not t.is_cuda:
        if not t.is_pinned():
            raise ValueError(f"{name}: a host tensor must be pinned (page-locked)")
        if not t.is_contiguous():
            raise ValueError(f"{name}: must be contiguous")
        if dtypes is not None and t.dtype not in dtypes:
            raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
        if numel is not None and t.numel() < numel:
            raise ValueError(f"{name}: has {t.numel()} elements, needs {numel}")
        return t.data_ptr()
    return _ptr(t, name, dtypes, numel)


def _pool_args(k_data, k_scale, v_data, v_scale, host: bool):
    f = _hptr if host else _ptr
    return (f(k_data, "k_data", (torch.uint8,)), f(k_scale, "k_scale", _U16), f(v_data, "v_data", (torch.uint8,)),
            f(v_scale, "v_scale", _U16))


def qkv_stage_pages_f4(dst_k_data, dst_k_scale, dst_v_data, dst_v_scale, src_k_data, src_k_scale, src_v_data,
                       src_v_scale, src_pages, dst_page0: int = 0, device_status=None, stream=None):
    """Copy source pages src_pages[i] (int32, device or pinned host) into
    destination pages dst_page0 + i. The source pool may be pinned host
    memory (read over the host link) or device memory."""
    num_pages, kv_heads, block_size, half = dst_k_data.shape
    head_dim = 2 * half
    if tuple(src_k_data.shape[1:]) != (kv_heads, block_size, half) or src_v_scale.shape[1:] != dst_v_scale.shape[1:]:
        raise ValueError("source and destination pools must have the same page shape")
    n = src_pages.numel()
    _check("qkv_stage_pages_f4", lib.qkv_stage_pages_f4(
        *_pool_args(dst_k_data, dst_k_scale, dst_v_data, dst_v_scale, False), num_pages, int(dst_page0),
        *_pool_args(src_k_data, src_k_scale, src_v_data, src_v_scale, True), src_k_data.shape[0],
        _hptr(src_pages, "src_pages", (torch.int32,)), n, kv_heads, head_dim, block_size,
        v_group_of(dst_v_scale, head_dim), _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def qkv_paged_decode_tiered_workspace_bytes(q_heads: int, kv_heads: int, head_dim: int, block_size: int,
                                            v_group: int, max_host_pages_per_seq: int, window_pages: int,
                                            max_splits: int) -> int:
    return lib.qkv_paged_decode_tiered_workspace_bytes(int(q_heads), int(kv_heads), int(head_dim), int(block_size),
                                                       int(v_group), int(max_host_pages_per_seq), int(window_pages),
                                                       int(max_splits))


def qkv_paged_decode_attn_f4_tiered(out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, host_k_data,
                                    host_k_scale, host_v_data, host_v_scale, host_page_table, host_lens,
                                    kv_heads: int, window_pages: int, max_splits: int, workspace, lse2_out=None,
                                    softmax_scale: float = 0.0, device_status=None, stream=None):
    """Decode attention over host_lens[s] tokens of the pinned host pool
    (pages host_page_table[s]) followed by seq_lens[s] tokens of the device
    pool (pages page_table[s]). host_lens: host integers (a list, numpy array
    or CPU tensor), whole pages. workspace: a uint8 CUDA tensor of
    qkv_paged_decode_tiered_workspace_bytes(...) bytes."""
    n_seq, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    hl = np.ascontiguousarray(np.asarray(host_lens.cpu() if isinstance(host_lens, torch.Tensor) else host_lens,
                                         dtype=np.int32))
    if hl.size != n_seq:
        raise ValueError(f"host_lens: {hl.size} entries for {n_seq} sequences")
    _check("qkv_paged_decode_attn_f4_tiered", lib.qkv_paged_decode_attn_f4_tiered(
        _ptr(out, "out", _U16, n_seq * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,), n_seq * q_heads),
        _ptr(q, "q", _U16), *_pool_args(k_data, k_scale, v_data, v_scale, False),
        _ptr(page_table, "page_table", (torch.int32,)), _ptr(seq_lens, "seq_lens", (torch.int32,), n_seq),
        page_table.shape[1], num_pages, *_pool_args(host_k_data, host_k_scale, host_v_data, host_v_scale, True),
        host_k_data.shape[0], _hptr(host_page_table, "host_page_table", (torch.int32,), n_seq),
        host_page_table.shape[1], hl.ctypes.data, n_seq, q_heads, kv_heads, head_dim, block_size,
        v_group_of(v_scale, head_dim), float(softmax_scale), int(window_pages), int(max_splits),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _ptr(device_status, "device_status", (torch.int32,)), _stream(stream)))


def qkv_paged_prefill_auto_splits(n_q: int, prefix_len: int, q_heads: int, kv_heads: int, head_dim: int,
                                  workspace_bytes: int) -> int:
    return lib.qkv_paged_prefill_auto_splits(int(n_q), int(prefix_len), int(q_heads), int(kv_heads), int(head_dim),
                                             int(workspace_bytes))


def qkv_paged_prefill_tiered_workspace_bytes(n_q: int, q_heads: int, kv_heads: int, head_dim: int, block_size: int,
                                             v_group: int, max_host_pages: int, window_pages: int,
                                             parts_per_launch: int) -> int:
    return lib.qkv_paged_prefill_tiered_workspace_bytes(int(n_q), int(q_heads), int(kv_heads), int(head_dim),
                                                        int(block_size), int(v_group), int(max_host_pages),
                                                        int(window_pages), int(parts_per_launch))


def qkv_paged_prefill_attn_f4_tiered(out, q, k_data, k_scale, v_data, v_scale, page_table, prefix_len: int,
                                     host_k_data, host_k_scale, host_v_data, host_v_scale, host_page_table,
                                     host_len: int, kv_heads: int, window_pages: int, parts_per_launch: int,
                                     workspace, lse2_out=None, softmax_scale: float = 0.0, device_status=None,
                                     stream=None):
    """Chunked causal prefill of one sequence whose first host_len tokens
    (whole pages, pages host_page_table) sit in the pinned host pool; the rest
    of its context, the chunk included, in the device pool (row page_table,
    the chunk at device tokens prefix_len .. prefix_len + n_q - 1)."""
    n_q, q_heads, head_dim = q.shape
    num_pages, _, block_size, _ = k_data.shape
    page_table = page_table.reshape(-1)
    host_page_table = host_page_table.reshape(-1)
    _check("qkv_paged_prefill_attn_f4_tiered", lib.qkv_paged_prefill_attn_f4_tiered(
        _ptr(out, "out", _U16, n_q * q_heads * head_dim), _ptr(lse2_out, "lse2_out", (torch.float32,), n_q * q_heads),
        _ptr(q, "q", _U16), *_pool_args(k_data, k_scale, v_data, v_scale, False),
        _ptr(page_table, "page_table", (torch.int32,)), n_q, int(prefix_len), page_table.numel(), num_pages,
        *_pool_args(host_k_data, host_k_scale, host_v_data, host_v_scale, True), host_k_data.shape[0],
        _hptr(host_page_table, "host_page_table", (torch.int32,), int(host_len) // block_size), int(host_len),
        q_heads, kv_heads, head_dim, block_size, v_group_of(v_scale, head_dim), float(softmax_scale),
        int(window_pages), int(parts_per_launch), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _ptr(device_status, "device_status", (torch.int32,)),
        _stream(stream)))
