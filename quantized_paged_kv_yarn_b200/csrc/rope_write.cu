// rope_write.cu -- partial rotary of q and the new k, and the F4 write of the
// new k and v, in one launch (sm_100a).
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 1
// (YaRN partial rotary) and section 2 (reshape-and-cache F4 write); ignis docs
// "context-and-speculation", --model-rope-scaling (the attention factor on
// queries and keys alike).
//
// The arithmetic is that of qkv_rope_apply followed by qkv_kv_write_f4: the
// rotated k is rounded to bf16 before it is quantised, so the cache bytes are
// identical to the two-call path.
#include "common.cuh"

namespace qkv {

// Warp items per token: [0, Hq) rotate a q head; [Hq, Hq + Hkv) rotate a k
// head and write its F4 row; [Hq + Hkv, Hq + 2 Hkv) write a v head's F4 row.
__global__ void __launch_bounds__(256) rope_kv_write_kernel(
    const __nv_bfloat16* q_in, __nv_bfloat16* q_out,  // may alias
    const uint16_t* __restrict__ k_in, const uint16_t* __restrict__ v_in, uint16_t* __restrict__ k_out,
    const int64_t* __restrict__ positions, const int64_t* __restrict__ slots, int n_tok, int q_heads,
    int kv_heads, int head_dim, int rot, const float* __restrict__ cos_tab, const float* __restrict__ sin_tab,
    int64_t tab_start, int64_t tab_len, uint8_t* __restrict__ k_data, __half* __restrict__ k_scale,
    uint8_t* __restrict__ v_data, __half* __restrict__ v_scale, int block, int64_t num_pages, int v_group,
    int32_t* status) {
  pdl_wait();  // writes the cache: no early start of its successor
  const int lane = threadIdx.x & 31;
  const int per_tok = q_heads + 2 * kv_heads;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= (int64_t)n_tok * per_tok) return;
  const int64_t tok = item / per_tok;
  const int kind = (int)(item - tok * per_tok);
  const int half = rot / 2;
  const int64_t row = positions[tok] - tab_start;
  const bool pos_ok = row >= 0 && row < tab_len;

  if (kind < q_heads) {  // ---- rotary of one q head (as qkv_rope_apply)
    const __nv_bfloat16* xi = q_in + (tok * q_heads + kind) * head_dim;
    __nv_bfloat16* xo = q_out + (tok * q_heads + kind) * head_dim;
    if (!pos_ok && lane == 0 && kind == 0) flag(status, QKV_DEV_BAD_POSITION);
    for (int j = lane; j < half; j += 32) {
      const float x0 = __bfloat162float(xi[j]), x1 = __bfloat162float(xi[j + half]);
      if (pos_ok) {
        const float c = cos_tab[row * half + j], s = sin_tab[row * half + j];
        xo[j] = __float2bfloat16_rn(rot_first(x0, x1, c, s));
        xo[j + half] = __float2bfloat16_rn(rot_second(x0, x1, c, s));
      } else {
        xo[j] = xi[j];
        xo[j + half] = xi[j + half];
      }
    }
    if (xi != xo)
      for (int j = rot + lane; j < head_dim; j += 32) xo[j] = xi[j];
    return;
  }

  // ---- one k or v head row: lane l holds elements 8l .. 8l+7
  const bool is_k = kind < q_heads + kv_heads;
  const int h = is_k ? kind - q_heads : kind - q_heads - kv_heads;
  float x[8];
  load_row8((is_k ? k_in : v_in) + (tok * kv_heads + h) * head_dim, lane, head_dim, x);
  if (is_k) {
    if (pos_ok) rope_row_bf16(x, lane, rot, cos_tab + row * half, sin_tab + row * half);
    if (!pos_ok && lane == 0 && h == 0) flag(status, QKV_DEV_BAD_POSITION);
    if (k_out && lane * 8 < head_dim) {
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) ow[i] = (__float_as_uint(x[2 * i]) >> 16) | (__float_as_uint(x[2 * i + 1]) & 0xffff0000u);
      *reinterpret_cast<uint4*>(k_out + (tok * kv_heads + h) * head_dim + lane * 8) = o;
    }
  }

  // ---- F4 quantise-write (as qkv_kv_write_f4)
  const int64_t slot = slots[tok];
  if (slot < 0) return;
  if (slot >= num_pages * block) {
    if (lane == 0 && is_k && h == 0) flag(status, QKV_DEV_BAD_SLOT);
    return;
  }
  const int group = is_k ? 32 : v_group;
  const int64_t page = slot / block, off = slot - page * block;
  const int64_t crow = (page * kv_heads + h) * block + off;
  f4_write_row(x, lane, head_dim, group, (is_k ? k_data : v_data) + crow * (head_dim / 2),
               (is_k ? k_scale : v_scale) + crow * (head_dim / group));
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_rope_kv_write_f4_v(const uint16_t* q_in, uint16_t* q_out, const uint16_t* k_in,
                                      const uint16_t* v_in, uint16_t* k_out, const int64_t* positions,
                                      const int64_t* slot_mapping, int32_t n_tok, int32_t q_heads,
                                      int32_t kv_heads, int32_t head_dim, int32_t rot_dim, const float* cos_tab,
                                      const float* sin_tab, int64_t table_pos_start, int64_t table_len,
                                      uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                                      int32_t block_size, int64_t num_pages, int32_t v_group,
                                      int32_t* device_status, qkv_stream_t stream) {
  if (n_tok == 0) return QKV_OK;
  if (!q_in || !q_out || !k_in || !v_in || !positions || !slot_mapping || !cos_tab || !sin_tab || !k_data ||
      !k_scale || !v_data || !v_scale)
    return QKV_EINVAL;
  if (n_tok < 0 || q_heads < 0 || kv_heads < 1 || head_dim < 32 || head_dim > 256 || head_dim % 32 ||
      rot_dim < 16 || rot_dim % 16 || rot_dim > head_dim || table_len < 0 || block_size < 1 || num_pages < 1 ||
      (v_group != 32 && v_group != head_dim))
    return QKV_EINVAL;
  if (((uintptr_t)k_in | (uintptr_t)v_in | (uintptr_t)k_out) & 15) return QKV_EINVAL;
  if (((uintptr_t)k_data | (uintptr_t)v_data) & 3) return QKV_EINVAL;
  if (((uintptr_t)k_scale | (uintptr_t)v_scale) & 1) return QKV_EINVAL;
  if (q_in != q_out) {
    const size_t bytes = (size_t)n_tok * q_heads * head_dim * 2;
    const char *a = (const char*)q_in, *b = (const char*)q_out;
    if (a < b + bytes && b < a + bytes) return QKV_EINVAL;
  }
  const int64_t warps = (int64_t)n_tok * (q_heads + 2 * kv_heads);
  const int64_t blocks = (warps + 7) / 8;
  if (blocks > 0x7fffffff) return QKV_EINVAL;
  const __nv_bfloat16* qi = reinterpret_cast<const __nv_bfloat16*>(q_in);
  __nv_bfloat16* qo = reinterpret_cast<__nv_bfloat16*>(q_out);
  __half* ks = reinterpret_cast<__half*>(k_scale);
  __half* vs = reinterpret_cast<__half*>(v_scale);
  int nt = n_tok, hq = q_heads, hkv = kv_heads, hd = head_dim, rd = rot_dim, bs = block_size, vg = v_group;
  void* args[] = {&qi, &qo, &k_in, &v_in, &k_out, &positions, &slot_mapping, &nt, &hq, &hkv, &hd, &rd,
                  &cos_tab, &sin_tab, &table_pos_start, &table_len, &k_data, &ks, &v_data, &vs, &bs, &num_pages,
                  &vg, &device_status};
  if (launch_pdl((const void*)rope_kv_write_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, args) !=
      cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" int qkv_rope_kv_write_f4(const uint16_t* q_in, uint16_t* q_out, const uint16_t* k_in,
                                    const uint16_t* v_in, uint16_t* k_out, const int64_t* positions,
                                    const int64_t* slot_mapping, int32_t n_tok, int32_t q_heads,
                                    int32_t kv_heads, int32_t head_dim, int32_t rot_dim, const float* cos_tab,
                                    const float* sin_tab, int64_t table_pos_start, int64_t table_len,
                                    uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                                    int32_t block_size, int64_t num_pages, int32_t* device_status,
                                    qkv_stream_t stream) {
  return qkv_rope_kv_write_f4_v(q_in, q_out, k_in, v_in, k_out, positions, slot_mapping, n_tok, q_heads, kv_heads,
                                head_dim, rot_dim, cos_tab, sin_tab, table_pos_start, table_len, k_data, k_scale,
                                v_data, v_scale, block_size, num_pages, 32, device_status, stream);
}
