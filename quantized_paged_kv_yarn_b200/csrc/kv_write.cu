// kv_write.cu -- quantise new K/V rows into the paged F4 cache (sm_100a).
//
// Source: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2:
// a reshape-and-cache kernel writes symmetric 4-bit values
// (nibble - 8) * scale through a slot mapping, one scale per 32-value K cell
// and "one scale per token per V head" (v_group = head_dim; v_group = 32
// gives V the K layout).
//
// Exactness. The scale is amax / 7 rounded once to fp16 and the code is
// rint(x / scale). Both divisions run in IEEE float (correctly rounded), and
// that decides every rounding exactly as exact division would:
//  * x (bf16, 8 significant bits) / scale (fp16, 11 bits): an inexact
//    quotient of magnitude <= 8.5 lies at least 2^-20 from every half-integer,
//    while float rounding moves it by at most 8.5 * 2^-24; exact half-integer
//    quotients are representable and round to even in rintf.
//    (The same holds for a V group of head_dim values.)
//  * amax / 7 is never a dyadic rational unless 7 divides amax's significand
//    (then it is exact in float); otherwise it lies at least ulp16 / 14 from
//    every fp16 rounding midpoint, far beyond float's 2^-24 relative error.
#include "common.cuh"

namespace qkv {

// One warp per (token, kv head, K or V). Lane l holds elements 8l .. 8l+7,
// so four lanes form one 32-value cell (v_group / 8 lanes one V group) and
// the warp stores 128 contiguous bytes of packed nibbles.
__global__ void __launch_bounds__(256) kv_write_f4_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, const int64_t* __restrict__ slots,
    int n_tok, uint8_t* __restrict__ k_data, __half* __restrict__ k_scale, uint8_t* __restrict__ v_data,
    __half* __restrict__ v_scale, int kv_heads, int head_dim, int block, int64_t num_pages, int v_group,
    int32_t* status) {
  pdl_wait();  // writes the cache: no early start of its successor
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= (int64_t)n_tok * kv_heads * 2) return;
  const int which = (int)(item & 1);
  const int64_t th = item >> 1;
  const int64_t tok = th / kv_heads;
  const int h = (int)(th - tok * kv_heads);
  const int64_t slot = slots[tok];
  if (slot < 0) return;
  if (slot >= num_pages * block) {
    if (lane == 0 && which == 0 && h == 0) flag(status, QKV_DEV_BAD_SLOT);
    return;
  }
  const int64_t page = slot / block, off = slot - page * block;
  const bool active = lane * 8 < head_dim;
  const uint16_t* src = (which ? v : k) + (tok * kv_heads + h) * head_dim;

  float x[8];
  float amax = 0.f;
  if (active) {
    const uint4 raw = *reinterpret_cast<const uint4*>(src + lane * 8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  }
  // Lanes per scale group: 4 for a 32-value cell; the whole warp for a V
  // group of head_dim values (lanes past head_dim / 8 hold amax 0).
  const int group = which ? v_group : 32;
  const int gl = group == 32 ? 4 : 32;
  for (int o = 1; o < gl; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL_MASK, amax, o));
  if (!active) return;

  const __half sh = __float2half_rn(fminf(__fdiv_rn(amax, 7.0f), 65504.0f));
  const float s = __half2float(sh);
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int code = 8;
    if (s != 0.f) code = (int)fminf(7.f, fmaxf(-8.f, rintf(__fdiv_rn(x[i], s)))) + 8;
    word |= (uint32_t)code << (4 * i);
  }
  const int64_t row = (page * kv_heads + h) * block + off;
  uint8_t* dst = (which ? v_data : k_data) + row * (head_dim / 2);
  reinterpret_cast<uint32_t*>(dst)[lane] = word;
  if ((lane & (gl - 1)) == 0) (which ? v_scale : k_scale)[row * (head_dim / group) + lane / gl] = sh;
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_kv_write_f4_v(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping,
                                 int32_t n_tok, uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data,
                                 uint16_t* v_scale, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                 int64_t num_pages, int32_t v_group, int32_t* device_status, qkv_stream_t stream) {
  if (n_tok == 0) return QKV_OK;  // nothing to read or write; pointers may be NULL
  if (!k || !v || !slot_mapping || !k_data || !k_scale || !v_data || !v_scale) return QKV_EINVAL;
  if (n_tok < 0 || kv_heads < 1 || head_dim < 32 || head_dim > 256 || head_dim % 32 || block_size < 1 ||
      num_pages < 1 || (v_group != 32 && v_group != head_dim))
    return QKV_EINVAL;
  if (((uintptr_t)k | (uintptr_t)v) & 15) return QKV_EINVAL;
  if (((uintptr_t)k_data | (uintptr_t)v_data) & 3) return QKV_EINVAL;
  if (((uintptr_t)k_scale | (uintptr_t)v_scale) & 1) return QKV_EINVAL;
  const int64_t warps = (int64_t)n_tok * kv_heads * 2;
  if (warps == 0) return QKV_OK;
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffff) return QKV_EINVAL;
  __half* ks = reinterpret_cast<__half*>(k_scale);
  __half* vs = reinterpret_cast<__half*>(v_scale);
  int nt = n_tok, kvh = kv_heads, hd = head_dim, bs = block_size, vg = v_group;
  void* args[] = {&k, &v, &slot_mapping, &nt, &k_data, &ks, &v_data, &vs, &kvh, &hd, &bs, &num_pages, &vg,
                  &device_status};
  if (launch_pdl((const void*)kv_write_f4_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" int qkv_kv_write_f4(const uint16_t* k, const uint16_t* v, const int64_t* slot_mapping, int32_t n_tok,
                               uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                               int32_t kv_heads, int32_t head_dim, int32_t block_size, int64_t num_pages,
                               int32_t* device_status, qkv_stream_t stream) {
  return qkv_kv_write_f4_v(k, v, slot_mapping, n_tok, k_data, k_scale, v_data, v_scale, kv_heads, head_dim,
                           block_size, num_pages, 32, device_status, stream);
}
