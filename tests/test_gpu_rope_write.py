"""GPU parity of the YaRN table, the partial rotary and the F4 write against
the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import to_dev, to_host

pytestmark = pytest.mark.gpu

YARN4 = dict(rope_base=1e7, rot_dim=64, factor=4.0, orig_max_pos=262144, beta_fast=32.0, beta_slow=1.0)
PLAIN = dict(rope_base=1e7, rot_dim=64, factor=1.0)
SPECS = {"yarn4": YARN4, "plain": PLAIN, "yarn1.22": dict(YARN4, factor=1.220703125),
         "yarn_rot128": dict(YARN4, rot_dim=128), "yarn_ext0": dict(YARN4, ext_factor=0.0)}


@pytest.fixture(scope="module")
def qkv():
    import quantized_paged_kv_yarn_b200 as q
    return q


def _params(qkv, spec):
    return qkv.YarnParams.make(**spec)


def _table(qkv, spec, pos0, n):
    h = spec["rot_dim"] // 2
    c = torch.empty((n, h), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    qkv.qkv_yarn_rope_table(_params(qkv, spec), pos0, n, c, s)
    return c, s


@pytest.mark.parametrize("name", list(SPECS))
@pytest.mark.parametrize("pos0,n", [(0, 4096), (262144, 3), (319999, 1), (524287 - 1000, 1001), (1048575 - 7, 8)])
def test_yarn_table(qkv, name, pos0, n):
    spec = SPECS[name]
    c, s = _table(qkv, spec, pos0, n)
    torch.cuda.synchronize()
    rc, rs = oracle.yarn_table(spec, pos0, n)
    _, ms, _, _ = oracle.yarn_theta(spec)
    # tables within 1e-6 of the table scale (the values are bounded by it)
    assert np.max(np.abs(to_host(c) - rc)) <= 1e-6 * ms
    assert np.max(np.abs(to_host(s) - rs)) <= 1e-6 * ms


def test_yarn_table_empty_and_errors(qkv):
    c = torch.empty(256, device="cuda")
    qkv.qkv_yarn_rope_table(_params(qkv, YARN4), 0, 0, c, c)
    with pytest.raises(qkv.QkvError):
        qkv.qkv_yarn_rope_table(_params(qkv, dict(YARN4, rot_dim=63)), 0, 1, c, c)
    with pytest.raises(qkv.QkvError):
        qkv.qkv_yarn_rope_table(_params(qkv, dict(YARN4, factor=0.5)), 0, 1, c, c)


@pytest.mark.parametrize("inplace", [False, True])
@pytest.mark.parametrize("name", ["yarn4", "plain", "yarn_rot128"])
def test_rope_apply(qkv, name, inplace):
    spec = SPECS[name]
    rng = np.random.default_rng(11)
    n_tok, heads, d = 37, 16, 256
    x = workloads.f32_to_bf16_bits((rng.standard_normal((n_tok, heads, d)) * 3).astype(np.float32))
    pos = np.sort(rng.integers(262000, 1048576, n_tok)).astype(np.int64)
    pos[0], pos[-1] = 262000, 1048575
    p0 = int(pos.min())
    c, s = _table(qkv, spec, p0, int(pos.max()) - p0 + 1)
    xi = to_dev(x)
    xo = xi if inplace else torch.empty_like(xi)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_rope_apply(xi, xo, to_dev(pos), c, s, p0, spec["rot_dim"], device_status=st)
    got = to_host(xo, np.uint16)
    want = oracle.rope_apply_bf16(x, pos, spec)
    assert int(st.item()) == 0
    rot = spec["rot_dim"]
    assert np.array_equal(got[..., rot:], x[..., rot:])
    g = workloads.bf16_bits_to_f32(got[..., :rot]).astype(np.float64)
    w = workloads.bf16_bits_to_f32(want[..., :rot]).astype(np.float64)
    # float math on a float table vs double everywhere: at most one bf16 step
    from helpers import bf16_ulp
    assert np.all(np.abs(g - w) <= bf16_ulp(np.maximum(np.abs(g), np.abs(w))) * 1.0000001)
    assert np.mean(got == want) > 0.97


def test_rope_position_outside_table(qkv):
    x = to_dev(np.full((2, 1, 256), 0x3F80, np.uint16))
    c, s = _table(qkv, YARN4, 100, 10)
    out = torch.zeros_like(x)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_rope_apply(x, out, to_dev(np.array([105, 110], np.int64)), c, s, 100, 64, device_status=st)
    assert int(st.item()) == qkv.DEV_BAD_POSITION
    assert np.array_equal(to_host(out, np.uint16)[1], to_host(x, np.uint16)[1])


def _write_both(qkv, k, v, slots, num_pages, kv_heads, block, head_dim, v_group=32):
    cache = qkv.PagedF4Cache.allocate(num_pages, kv_heads, block, head_dim, v_group=v_group)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache.write(to_dev(k), to_dev(v), to_dev(slots), device_status=st)
    ref = oracle.empty_cache(num_pages, kv_heads, block, head_dim, v_group=v_group)
    bad = oracle.kv_write_f4(k, v, slots, ref, kv_heads, head_dim, block)
    got = (to_host(cache.k_data), to_host(cache.k_scale).view(np.uint16), to_host(cache.v_data),
           to_host(cache.v_scale).view(np.uint16))
    return got, ref, int(st.item()), bad


@pytest.mark.parametrize("v_group", [32, 0])
@pytest.mark.parametrize("head_dim", [256, 128, 96, 64])
def test_kv_write_bitexact(qkv, head_dim, v_group):
    """v_group 0 stands for head_dim: one V scale per token and head."""
    v_group = v_group or head_dim
    rng = np.random.default_rng(12)
    n_tok, kv_heads, block, num_pages = 300, 4, 16, 40
    x = rng.standard_normal((2, n_tok, kv_heads, head_dim)) * 10.0 ** rng.uniform(-6, 4, (2, n_tok, kv_heads, 1))
    x[0, 5] = 0.0                       # zero cells
    x[1, 6, :, :32] = 1e-9              # scale underflows
    x[0, 7, :, 3] = 3e38                # saturating scale
    x[1, 8] = np.round(x[1, 8])         # many exact ties
    x[0, 9, 0, :32] = (np.arange(32) - 16) * 0.5   # half-integers at scale 16/7
    k = workloads.f32_to_bf16_bits(x[0].astype(np.float32))
    v = workloads.f32_to_bf16_bits(x[1].astype(np.float32))
    slots = rng.permutation(num_pages * block)[:n_tok].astype(np.int64)
    slots[3] = -1
    got, ref, st, bad = _write_both(qkv, k, v, slots, num_pages, kv_heads, block, head_dim, v_group)
    assert st == 0 and bad == 0
    assert got[3].shape[-1] == head_dim // v_group
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


def test_kv_write_bad_slot(qkv):
    k = workloads.f32_to_bf16_bits(np.ones((2, 1, 256), np.float32))
    got, ref, st, bad = _write_both(qkv, k, k, np.array([3, 64 * 4], np.int64), 4, 1, 64, 256)
    assert st == qkv.DEV_BAD_SLOT and bad == 1
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("v_group", [32, 256])
@pytest.mark.parametrize("amax_bits", [0x3F80, 0x0080, 0x7F7F, 0x3380, 0x0001, 0x4B00])
def test_kv_write_exhaustive_bf16(qkv, amax_bits, v_group):
    """Every finite bf16 value as one element of a cell whose amax is fixed
    (with v_group 256 the V row's amax is the larger of the two)."""
    allb = np.arange(65536, dtype=np.uint16)
    vals = allb[(allb & 0x7F80) != 0x7F80]
    n = vals.size
    k = np.zeros((n, 1, 256), np.uint16)
    k[:, 0, 0] = amax_bits
    k[:, 0, 1] = vals
    k[:, 0, 32 + 7] = vals          # a second cell: the value alone sets amax
    got, ref, st, bad = _write_both(qkv, k, k, np.arange(n, dtype=np.int64), n // 64 + 1, 1, 64, 256, v_group)
    assert st == 0
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("v_group", [32, 256])
@pytest.mark.parametrize("inplace", [False, True])
@pytest.mark.parametrize("rot", [64, 128, 256])
def test_rope_kv_write_fused_matches_two_calls(qkv, rot, inplace, v_group):
    """The one-launch rotary + F4 write gives the same bits as qkv_rope_apply
    on q and k followed by qkv_kv_write_f4 (and so the oracle parity of those
    two calls carries over)."""
    spec = dict(YARN4, rot_dim=rot)
    rng = np.random.default_rng(13)
    n_tok, hq, hkv, d, B, P = 9, 16, 4, 256, 16, 12
    q = workloads.f32_to_bf16_bits((rng.standard_normal((n_tok, hq, d)) * 2).astype(np.float32))
    k = workloads.f32_to_bf16_bits((rng.standard_normal((n_tok, hkv, d)) * 3).astype(np.float32))
    v = workloads.f32_to_bf16_bits(rng.standard_normal((n_tok, hkv, d)).astype(np.float32))
    pos = np.sort(rng.integers(262144, 1048576, n_tok)).astype(np.int64)
    slots = rng.permutation(P * B)[:n_tok].astype(np.int64)
    slots[2] = -1
    p0 = int(pos.min())
    c, s = _table(qkv, spec, p0, int(pos.max()) - p0 + 1)
    # two calls
    q2 = torch.empty_like(to_dev(q))
    k2 = torch.empty_like(to_dev(k))
    qkv.qkv_rope_apply(to_dev(q), q2, to_dev(pos), c, s, p0, rot)
    qkv.qkv_rope_apply(to_dev(k), k2, to_dev(pos), c, s, p0, rot)
    ref = qkv.PagedF4Cache.allocate(P, hkv, B, d, v_group=v_group)
    ref.write(k2, to_dev(v), to_dev(slots))
    # one launch
    qi = to_dev(q)
    qo = qi if inplace else torch.empty_like(qi)
    ko = torch.empty_like(to_dev(k))
    got = qkv.PagedF4Cache.allocate(P, hkv, B, d, v_group=v_group)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_rope_kv_write_f4(qi, qo, to_dev(k), to_dev(v), to_dev(pos), to_dev(slots), c, s, p0, rot, got.k_data,
                             got.k_scale, got.v_data, got.v_scale, k_out=ko, device_status=st)
    assert int(st.item()) == 0
    assert torch.equal(qo, q2) and torch.equal(ko, k2)
    for a, b in zip((got.k_data, got.k_scale, got.v_data, got.v_scale), (ref.k_data, ref.k_scale, ref.v_data,
                                                                          ref.v_scale)):
        assert torch.equal(a, b)


def test_rope_kv_write_fused_flags(qkv):
    k = to_dev(np.full((2, 1, 256), 0x3F80, np.uint16))
    q = to_dev(np.full((2, 2, 256), 0x3F80, np.uint16))
    c, s = _table(qkv, YARN4, 100, 10)
    cache = qkv.PagedF4Cache.allocate(2, 1, 16, 256)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qkv.qkv_rope_kv_write_f4(q, q, k, k, to_dev(np.array([105, 200], np.int64)), to_dev(np.array([3, 32], np.int64)),
                             c, s, 100, 64, cache.k_data, cache.k_scale, cache.v_data, cache.v_scale,
                             device_status=st)
    assert int(st.item()) == qkv.DEV_BAD_POSITION | qkv.DEV_BAD_SLOT
