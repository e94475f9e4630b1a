"""B200 (sm_100a) decode hot path over a paged 4-bit K/V cache with YaRN
partial rotary: a C-ABI CUDA library (``libqkv.so``, declared in
``include/qkv.h``) and this thin ctypes binding.

The binding only marshals arguments: it checks tensor dtypes, shapes,
devices and contiguity, passes raw pointers and the current CUDA stream, and
raises :class:`QkvError` on a non-zero return code. All computation runs in
the library's kernels; there is no CPU fallback. If the library is missing,
importing this package raises.
"""
from ._abi import (  # noqa: F401
    LIB_PATH,
    QkvError,
    YarnParams,
    DEV_BAD_PAGE,
    DEV_BAD_POSITION,
    DEV_BAD_SEQLEN,
    DEV_BAD_SLOT,
    DEV_TIMEOUT,
    exported_symbols,
    lib,
    qkv_decode_step_f4,
    qkv_decode_step_split_f4,
    qkv_gather_kv_f4,
    qkv_kv_write_f4,
    qkv_lse_merge,
    qkv_paged_decode_attn_f4,
    qkv_paged_decode_attn_f4_static,
    qkv_paged_decode_attn_f4_tiered,
    qkv_paged_decode_tiered_workspace_bytes,
    STATIC_SCRATCH_BYTES,
    qkv_paged_decode_auto_splits,
    qkv_paged_decode_split_f4,
    qkv_paged_decode_workspace_bytes,
    qkv_paged_prefill_attn_f4,
    qkv_paged_prefill_attn_f4_tiered,
    qkv_paged_prefill_auto_splits,
    qkv_paged_prefill_tiered_workspace_bytes,
    qkv_paged_prefill_workspace_bytes,
    qkv_rope_apply,
    qkv_rope_kv_write_f4,
    qkv_stage_pages_f4,
    qkv_status_string,
    qkv_yarn_auto_factor,
    qkv_yarn_rope_table,
    v_group_of,
)
from .cache import DecodeAttention, PagedF4Cache, TieredDecodeAttention, TieredPrefillAttention  # noqa: F401
