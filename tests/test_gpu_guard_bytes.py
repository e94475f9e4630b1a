"""Guard bytes around the caller's buffers: every buffer the path writes (the
F4 cache, the YaRN table, the rotary output, the decode attention's output,
lse2 and workspace, the merge, the chunked prefill with and without a
context split, the gather) is passed as a view into a larger device buffer
whose bytes before and after the view hold a fixed pattern. The pattern
must come back unchanged, and the view must get the same bits as a plain
buffer given the same call. (No device sanitizer runs on this GPU pool; this
is the check that no kernel writes outside what it is given.)"""
import numpy as np
import pytest
import torch

import workloads
from helpers import oracle_layer, to_dev, to_host

pytestmark = pytest.mark.gpu

GUARD = 4096   # bytes on each side: a multiple of 256, so a view keeps every alignment the ABI asks for
PATTERN = 0xA5
YARN4 = dict(rope_base=1e7, rot_dim=64, factor=4.0, orig_max_pos=262144, beta_fast=32.0, beta_slow=1.0)


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


class Guarded:
    """A device buffer laid out as [GUARD pattern bytes | view | GUARD pattern bytes]."""

    def __init__(self, shape, dtype, device="cuda"):
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = int(np.prod(shape)) * esz
        self.raw = torch.full((self.nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=device)
        self.view = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def intact(self) -> bool:
        h = to_host(self.raw)
        return bool(np.all(h[:GUARD] == PATTERN) and np.all(h[GUARD + self.nbytes:] == PATTERN))


def _same(a, b):
    return np.array_equal(to_host(a).view(np.uint8), to_host(b).view(np.uint8))


def _guarded_cache(qkv, shape_like):
    """A PagedF4Cache whose four arrays are zeroed guarded views shaped like shape_like's."""
    gs = []
    for t in (shape_like.k_data, shape_like.k_scale, shape_like.v_data, shape_like.v_scale):
        g = Guarded(tuple(t.shape), t.dtype)
        g.view.zero_()
        gs.append(g)
    return gs, qkv.PagedF4Cache(*(g.view for g in gs))


def _filled_cache(qkv, w, x, cache):
    cache.write(to_dev(x["k_cache"]), to_dev(x["v_cache"]), to_dev(x["cache_slots"]))
    cache.write(to_dev(x["k_new"]), to_dev(x["v_new"]), to_dev(x["step_slots"]))
    return cache


def _decode_workload():
    return workloads.small("guard", seq_lens=(1000, 31, 4097), num_pages=200, block_size=32, q_heads=32,
                           kv_heads=4, page_alloc="interleaved", head_scale=True)


@pytest.mark.parametrize("v_group", [32, 256])
def test_kv_write_stays_in_the_cache(qkv, v_group):
    w = _decode_workload()
    x, _ = oracle_layer(w, v_group=v_group)
    plain = _filled_cache(qkv, w, x, qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim,
                                                                v_group=v_group))
    gs, cache = _guarded_cache(qkv, plain)
    _filled_cache(qkv, w, x, cache)
    torch.cuda.synchronize()
    for g, p in zip(gs, (plain.k_data, plain.k_scale, plain.v_data, plain.v_scale)):
        assert g.intact()
        assert _same(g.view, p)


def test_yarn_table_and_rotary_stay_in_their_outputs(qkv):
    params = qkv.YarnParams.make(**YARN4)
    p0, n_pos, h = 262000, 600, YARN4["rot_dim"] // 2
    c = torch.empty((n_pos, h), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    qkv.qkv_yarn_rope_table(params, p0, n_pos, c, s)
    gc, gsn = Guarded((n_pos, h), torch.float32), Guarded((n_pos, h), torch.float32)
    qkv.qkv_yarn_rope_table(params, p0, n_pos, gc.view, gsn.view)
    rng = np.random.default_rng(3)
    x = to_dev(workloads.f32_to_bf16_bits((rng.standard_normal((37, 16, 256)) * 3).astype(np.float32)))
    pos = to_dev(np.sort(rng.integers(p0, p0 + n_pos, 37)).astype(np.int64))
    plain = torch.empty_like(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_rope_apply(x, plain, pos, c, s, p0, YARN4["rot_dim"], device_status=st)
    gx = Guarded(tuple(x.shape), torch.int16)
    qkv.qkv_rope_apply(x, gx.view, pos, c, s, p0, YARN4["rot_dim"], device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for g, p in ((gc, c), (gsn, s), (gx, plain)):
        assert g.intact()
        assert _same(g.view, p)


def test_decode_attention_stays_in_its_outputs_and_workspace(qkv):
    w = _decode_workload()
    x, _ = oracle_layer(w)
    cache = _filled_cache(qkv, w, x, qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim))
    q, pt, sl = to_dev(x["q"]), to_dev(x["page_table"]), to_dev(x["seq_lens"])
    shape = (w.n_seq, w.q_heads, w.head_dim)
    att = qkv.DecodeAttention(w.n_seq, w.q_heads, w.kv_heads, w.head_dim, w.block_size)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    plain_o = torch.empty(shape, dtype=torch.int16, device="cuda")
    plain_l = torch.empty(shape[:2], dtype=torch.float32, device="cuda")
    att(plain_o, q, cache, pt, sl, lse2_out=plain_l, device_status=st)
    gws = Guarded(tuple(att.workspace.shape), torch.uint8)
    att.workspace = gws.view
    go, gl = Guarded(shape, torch.int16), Guarded(shape[:2], torch.float32)
    att(go.view, q, cache, pt, sl, lse2_out=gl.view, device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for g in (go, gl, gws):
        assert g.intact()
    assert _same(go.view, plain_o) and _same(gl.view, plain_l)


@pytest.mark.parametrize("n_parts", [5, 37])
def test_lse_merge_stays_in_its_outputs(qkv, n_parts):
    rng = np.random.default_rng(5 + n_parts)
    rows, d = 48, 256
    o = to_dev(rng.standard_normal((n_parts, rows, d)).astype(np.float32))
    l = to_dev((rng.standard_normal((n_parts, rows)) * 30).astype(np.float32))
    plain_o = torch.empty((rows, d), dtype=torch.int16, device="cuda")
    plain_l = torch.empty(rows, dtype=torch.float32, device="cuda")
    qkv.qkv_lse_merge(o, l, plain_o, plain_l)
    go, gl = Guarded((rows, d), torch.int16), Guarded((rows,), torch.float32)
    qkv.qkv_lse_merge(o, l, go.view, gl.view)
    torch.cuda.synchronize()
    assert go.intact() and gl.intact()
    assert _same(go.view, plain_o) and _same(gl.view, plain_l)


@pytest.mark.parametrize("splits", [1, 3])
def test_prefill_stays_in_its_outputs_and_workspace(qkv, splits):
    L, n_q, block, hq, hkv = 1600, 257, 32, 16, 4
    w = workloads.small("prefill", seq_lens=(L,), num_pages=-(-L // block) + 3, block_size=block, q_heads=hq,
                        kv_heads=hkv, head_scale=True, seed=0)
    x, _ = oracle_layer(w)
    cache = _filled_cache(qkv, w, x, qkv.PagedF4Cache.allocate(w.num_pages, hkv, block, 256))
    q = to_dev(workloads.chunk_queries_host(w, 0, n_q))
    pt = to_dev(np.ascontiguousarray(x["page_table"][0]))
    nb = qkv.qkv_paged_prefill_workspace_bytes(n_q, hq, 256, splits) if splits > 1 else 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def run(out, lse, ws):
        qkv.qkv_paged_prefill_attn_f4(out, q, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, pt, L - n_q,
                                      hkv, lse2_out=lse, num_splits=splits, workspace=ws, device_status=st)

    plain_o = torch.empty((n_q, hq, 256), dtype=torch.int16, device="cuda")
    plain_l = torch.empty((n_q, hq), dtype=torch.float32, device="cuda")
    run(plain_o, plain_l, torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None)
    go, gl = Guarded((n_q, hq, 256), torch.int16), Guarded((n_q, hq), torch.float32)
    gws = Guarded((nb,), torch.uint8) if nb else None
    run(go.view, gl.view, gws.view if gws else None)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for g in (go, gl) + ((gws,) if gws else ()):
        assert g.intact()
    assert _same(go.view, plain_o) and _same(gl.view, plain_l)


def test_gather_stays_in_its_outputs(qkv):
    w = _decode_workload()
    x, _ = oracle_layer(w)
    cache = _filled_cache(qkv, w, x, qkv.PagedF4Cache.allocate(w.num_pages, w.kv_heads, w.block_size, w.head_dim))
    lens = np.asarray(x["seq_lens"], np.int32)
    start = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    n_out = int(lens.sum())
    args = (to_dev(x["page_table"]), to_dev(lens), to_dev(start))
    shape = (n_out, w.kv_heads, w.head_dim)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pk = torch.empty(shape, dtype=torch.int16, device="cuda")
    pv = torch.empty_like(pk)
    qkv.qkv_gather_kv_f4(pk, pv, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, *args, device_status=st)
    gk, gv = Guarded(shape, torch.int16), Guarded(shape, torch.int16)
    qkv.qkv_gather_kv_f4(gk.view, gv.view, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale, *args,
                         device_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert gk.intact() and gv.intact()
    assert _same(gk.view, pk) and _same(gv.view, pv)
