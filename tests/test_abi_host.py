"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/qkv.h declares, and rejects invalid arguments before
launching anything."""
import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT, read_golden

HEADER = os.path.join(ROOT, "include", "qkv.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^QKV_API\s+[\w\s\*]+?\b(qkv_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def qkv():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import quantized_paged_kv_yarn_b200 as q
    return q


def test_exports_every_declared_symbol(qkv):
    declared = _declared()
    assert len(declared) >= 10
    lib = ctypes.CDLL(qkv.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(qkv.exported_symbols()) == declared


def test_auto_factor_rule_printed_examples(qkv):
    _, rows = read_golden("yarn_auto_factor.txt")
    for ctx, want in rows:
        got = qkv.qkv_yarn_auto_factor(int(ctx), 262144)
        assert got == float(want), (ctx, got, want)


def test_status_strings(qkv):
    assert qkv.qkv_status_string(0) == "ok"
    assert "invalid" in qkv.qkv_status_string(1)
    assert "unsupported" in qkv.qkv_status_string(2)
    assert qkv.qkv_status_string(99) == "unknown status"


def test_workspace_bytes(qkv):
    n = qkv.qkv_paged_decode_workspace_bytes(3, 16, 256, 74)
    rows = 3 * 16 * 74
    a = lambda x: (x + 255) // 256 * 256
    assert n == a(rows * 256 * 4) + a(rows * 4)   # o_parts, lse2_parts
    assert qkv.qkv_paged_decode_workspace_bytes(-1, 16, 256, 4) == 0



FAKE = ctypes.c_void_p(4096)  # never dereferenced: validation fails first
NUL = None


def test_invalid_arguments_rejected_before_launch(qkv):
    L = qkv.lib
    # rope table: odd rot_dim, factor < 1, null outputs
    p = qkv.YarnParams.make(rot_dim=63)
    assert L.qkv_yarn_rope_table(ctypes.byref(p), 0, 4, FAKE, FAKE, NUL) == 1
    p = qkv.YarnParams.make(factor=0.5)
    assert L.qkv_yarn_rope_table(ctypes.byref(p), 0, 4, FAKE, FAKE, NUL) == 1
    p = qkv.YarnParams.make()
    assert L.qkv_yarn_rope_table(ctypes.byref(p), 0, 4, NUL, FAKE, NUL) == 1
    assert L.qkv_yarn_rope_table(ctypes.byref(p), 0, 0, FAKE, FAKE, NUL) == 0   # nothing to do
    # rope apply: rot > head_dim, overlapping distinct buffers, empty
    assert L.qkv_rope_apply(FAKE, FAKE, FAKE, 1, 1, 64, 128, FAKE, FAKE, 0, 10, NUL, NUL) == 1
    assert L.qkv_rope_apply(ctypes.c_void_p(4096), ctypes.c_void_p(4098), FAKE, 1, 1, 64, 64, FAKE, FAKE, 0, 10,
                            NUL, NUL) == 1
    assert L.qkv_rope_apply(FAKE, FAKE, FAKE, 0, 16, 256, 64, FAKE, FAKE, 0, 10, NUL, NUL) == 0
    # kv write: head_dim not a multiple of 32, misaligned input, null cache
    assert L.qkv_kv_write_f4(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 4, 48, 64, 8, NUL, NUL) == 1
    assert L.qkv_kv_write_f4(ctypes.c_void_p(4098), FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 4, 256, 64, 8, NUL,
                             NUL) == 1
    assert L.qkv_kv_write_f4(FAKE, FAKE, FAKE, 1, NUL, FAKE, FAKE, FAKE, 4, 256, 64, 8, NUL, NUL) == 1
    assert L.qkv_kv_write_f4(FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, 4, 256, 64, 8, NUL, NUL) == 0
    # split pass: unsupported head_dim / group / block, bad group divisibility, null
    args = lambda hq, hkv, d, blk, ms=4: (FAKE, FAKE, ms, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, hq, hkv, d,
                                          blk, 16, 64, ctypes.c_float(0.0), 0, NUL, NUL)
    assert L.qkv_paged_decode_split_f4(*args(16, 4, 192, 64)) == 2     # head_dim: 256 and 128 are compiled
    assert L.qkv_paged_decode_split_f4(*args(16, 4, 64, 64)) == 2
    assert L.qkv_paged_decode_split_f4(*args(12, 4, 256, 64)) == 2     # group of 3
    assert L.qkv_paged_decode_split_f4(*args(16, 4, 256, 128)) == 2    # block 128
    assert L.qkv_paged_decode_split_f4(*args(16, 3, 256, 64)) == 1     # 16 % 3
    assert L.qkv_paged_decode_split_f4(*args(16, 4, 256, 64, 0)) == 1  # max_splits 0
    a = list(args(16, 4, 256, 64, 4)); a[18] = 5                       # num_splits above max_splits
    assert L.qkv_paged_decode_split_f4(*a) == 1
    a = list(args(16, 4, 256, 64)); a[3] = NUL
    assert L.qkv_paged_decode_split_f4(*a) == 1
    a = list(args(16, 4, 256, 64)); a[4] = ctypes.c_void_p(4100)       # cache not 16-byte aligned
    assert L.qkv_paged_decode_split_f4(*a) == 1
    # prefill: head_dim 256 and 128 are compiled (v_group = head_dim: one V scale per token)
    pf = lambda d: (FAKE, NUL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 0, 16, 4, d, 64, 16, 64,
                    ctypes.c_float(0.0), d, 1, NUL, 0, NUL, NUL)
    assert L.qkv_paged_prefill_attn_f4(*pf(192)) == 2
    assert L.qkv_paged_prefill_attn_f4(*pf(64)) == 2
    assert qkv.qkv_paged_prefill_auto_splits(64, 0, 16, 4, 192, 0) == 0
    # merge: bad head_dim, no parts, empty rows
    assert L.qkv_lse_merge(FAKE, FAKE, 4, 8, 30, FAKE, NUL, NUL) == 1
    assert L.qkv_lse_merge(FAKE, FAKE, 0, 8, 256, FAKE, NUL, NUL) == 1
    assert L.qkv_lse_merge(FAKE, FAKE, 4, 0, 256, FAKE, NUL, NUL) == 0
    # one-call attention: workspace too small or misaligned
    wa = lambda ws, nb: (FAKE, NUL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 16, 4, 256, 64, 16, 64,
                         ctypes.c_float(0.0), 0, 4, ws, nb, NUL, NUL)
    need = qkv.qkv_paged_decode_workspace_bytes(1, 16, 256, 4)
    assert L.qkv_paged_decode_attn_f4(*wa(FAKE, need - 1)) == 1
    assert L.qkv_paged_decode_attn_f4(*wa(ctypes.c_void_p(4096 + 16), need)) == 1


def test_tier_workspace_bytes(qkv):
    """Window (four page arrays), page table, count, then (windows + 1) *
    max_splits parts of q_heads * (head_dim + 1) floats, 256-byte aligned."""
    a = lambda x: (x + 255) // 256 * 256
    hq, hkv, d, blk, vg, max_host, win, ms = 16, 4, 256, 64, 32, 4096, 2048, 37
    rows = hkv * blk
    parts = (-(-max_host // win) + 1) * ms
    want = (2 * a(win * rows * d // 2) + a(win * rows * d // 32 * 2) + a(win * rows * d // vg * 2) + a(win * 4) + 256
            + a(parts * hq * d * 4) + a(parts * hq * 4))
    assert qkv.qkv_paged_decode_tiered_workspace_bytes(hq, hkv, d, blk, vg, max_host, win, ms) == want
    # per-token V scales shrink the V-scale window
    assert (qkv.qkv_paged_decode_tiered_workspace_bytes(hq, hkv, d, blk, d, max_host, win, ms)
            == want - a(win * rows * d // 32 * 2) + a(win * rows * 2))
    assert qkv.qkv_paged_decode_tiered_workspace_bytes(hq, hkv, d, blk, 48, max_host, win, ms) == 0
    assert qkv.qkv_paged_decode_tiered_workspace_bytes(hq, hkv, d, blk, vg, max_host, 0, ms) == 0


def test_tier_invalid_arguments_rejected_before_launch(qkv):
    L = qkv.lib
    i64 = ctypes.c_int64
    # staging: destination range past the pool, bad head_dim, pageable source
    st = lambda n, page0, d=256, src=FAKE: (FAKE, FAKE, FAKE, FAKE, i64(8), i64(page0), src, FAKE, FAKE, FAKE, i64(8),
                                            FAKE, n, 4, d, 64, 32, NUL, NUL)
    assert L.qkv_stage_pages_f4(*st(4, 5)) == 1
    assert L.qkv_stage_pages_f4(*st(4, -1)) == 1
    assert L.qkv_stage_pages_f4(*st(4, 0, d=48)) == 1
    assert L.qkv_stage_pages_f4(*st(0, 0)) == 0                         # nothing to do
    pageable = np.zeros(1 << 16, np.uint8)
    assert L.qkv_stage_pages_f4(*st(4, 0, src=ctypes.c_void_p(pageable.ctypes.data))) == 1
    # tiered decode: host lengths not whole pages or past the table, workspace too small
    need = qkv.qkv_paged_decode_tiered_workspace_bytes(16, 4, 256, 64, 32, 4, 2, 4)

    def td(host_lens, ws_bytes, host=FAKE):
        hl = np.asarray(host_lens, np.int32)
        return (FAKE, NUL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, i64(64), host, FAKE, FAKE, FAKE, i64(16),
                FAKE, 4, ctypes.c_void_p(hl.ctypes.data), len(hl), 16, 4, 256, 64, 32, ctypes.c_float(0.0), 2, 4,
                ctypes.c_void_p(1 << 20), ws_bytes, NUL, NUL), hl
    a, keep = td([64], need)
    assert L.qkv_paged_decode_attn_f4_tiered(*a) == 1              # FAKE host pool: not device-accessible
    a, keep = td([40], need)                                        # not whole pages
    assert L.qkv_paged_decode_attn_f4_tiered(*a) == 1
    a, keep = td([5 * 64], need)                                    # past max_host_pages_per_seq
    assert L.qkv_paged_decode_attn_f4_tiered(*a) == 1
    a, keep = td([64], need - 1)                                    # workspace too small
    assert L.qkv_paged_decode_attn_f4_tiered(*a) == 1
    a, keep = td([64], need, host=ctypes.c_void_p(pageable.ctypes.data))   # pageable host pool
    assert L.qkv_paged_decode_attn_f4_tiered(*a) == 1


def test_prefill_tier_workspace_bytes_and_refusals(qkv):
    a = lambda x: (x + 255) // 256 * 256
    n_q, hq, hkv, d, blk, vg, max_host, win, ppl = 2048, 16, 4, 256, 64, 32, 4032, 2048, 4
    rows = hkv * blk
    parts = (-(-max_host // win) + 1) * ppl
    want = (2 * a(win * rows * d // 2) + 2 * a(win * rows * d // 32 * 2) + a(win * 4) + 256
            + a(parts * n_q * hq * d * 4) + a(parts * n_q * hq * 4))
    assert qkv.qkv_paged_prefill_tiered_workspace_bytes(n_q, hq, hkv, d, blk, vg, max_host, win, ppl) == want
    assert qkv.qkv_paged_prefill_tiered_workspace_bytes(n_q, hq, hkv, d, blk, vg, max_host, win, 65) == 0
    assert qkv.qkv_paged_prefill_tiered_workspace_bytes(0, hq, hkv, d, blk, vg, max_host, win, ppl) == 0
    L = qkv.lib
    i64 = ctypes.c_int64
    need = qkv.qkv_paged_prefill_tiered_workspace_bytes(64, 16, 4, 256, 64, 32, 2, 2, 2)
    pageable = np.zeros(1 << 16, np.uint8)

    def tp(host_len, ws_bytes, host=FAKE):
        return (FAKE, NUL, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 0, 4, i64(64), host, FAKE, FAKE, FAKE, i64(16),
                FAKE, host_len, 16, 4, 256, 64, 32, ctypes.c_float(0.0), 2, 2, ctypes.c_void_p(1 << 20), ws_bytes,
                NUL, NUL)
    assert L.qkv_paged_prefill_attn_f4_tiered(*tp(40, need)) == 1          # host part not whole pages
    assert L.qkv_paged_prefill_attn_f4_tiered(*tp(128, need - 1)) == 1     # workspace too small
    assert L.qkv_paged_prefill_attn_f4_tiered(*tp(128, need)) == 1         # FAKE host pool: not device-accessible
    assert L.qkv_paged_prefill_attn_f4_tiered(*tp(128, need, ctypes.c_void_p(pageable.ctypes.data))) == 1
