// gather.cu -- the paged F4 cache read back into contiguous bf16 rows (sm_100a).
//
// Source: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2:
// gather_kv_cache gains an F4 path, i.e. the cache of a sequence is
// dequantised into contiguous rows for attention outside the paged kernels.
//
// Exactness: (code - 8) * scale needs at most 4 + 11 significant bits and is
// exact in float; one round-to-nearest-even to bf16 follows.
//
// Bound by HBM: 144 bytes read (one 128-byte packed row and its scales) and
// 512 bytes written per (token, KV head) for each of K and V. One thread per
// 32-value cell: a 16-byte load of its packed bytes, four 16-byte stores.
#include "common.cuh"

namespace qkv {

__global__ void __launch_bounds__(256) gather_kv_f4_kernel(
    const uint8_t* __restrict__ k_data, const __half* __restrict__ k_scale, const uint8_t* __restrict__ v_data,
    const __half* __restrict__ v_scale, const int32_t* __restrict__ page_table, int max_pages,
    const int32_t* __restrict__ seq_lens, const int64_t* __restrict__ out_start, int kv_heads, int head_dim,
    int block, int64_t num_pages, int v_group, int64_t n_out, uint16_t* __restrict__ k_out,
    uint16_t* __restrict__ v_out, int32_t* status) {
  pdl_release();
  pdl_wait();
  const int s = blockIdx.y;
  const int cells = head_dim / 32;
  // thread -> (token t, head h, K or V, cell c), cells fastest
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;  // < 2^31 (checked on the host)
  const uint32_t per_tok = (uint32_t)(kv_heads * 2 * cells);
  const int t = (int)(i / per_tok);
  int rem = (int)(i - (uint32_t)t * per_tok);
  const int h = rem / (2 * cells);
  rem -= h * 2 * cells;
  const int which = rem / cells, c = rem - which * cells;

  int len = seq_lens[s];
  const int64_t cap = (int64_t)max_pages * block;
  if (len < 0 || len > cap) {
    if (i == 0) flag(status, QKV_DEV_BAD_SEQLEN);
    len = len < 0 ? 0 : (int)cap;
  }
  if (t >= len) return;
  const int64_t orow = out_start[s] + t;
  if (orow < 0 || orow >= n_out) {
    if (rem == 0 && h == 0) flag(status, QKV_DEV_BAD_SEQLEN);
    return;
  }
  uint4* dst = reinterpret_cast<uint4*>((which ? v_out : k_out) + (orow * kv_heads + h) * head_dim + 32 * c);
  const int32_t page = page_table[(int64_t)s * max_pages + t / block];
  if (page < 0 || page >= num_pages) {
    if (t % block == 0 && rem == 0 && h == 0) flag(status, QKV_DEV_BAD_PAGE);
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < 4; ++j) __stcs(dst + j, z);
    return;
  }
  const int64_t row = ((int64_t)page * kv_heads + h) * block + t % block;
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>((which ? v_data : k_data) + row * (head_dim / 2)) + c);
  const int group = which ? v_group : 32;
  const float sc = __half2float((which ? v_scale : k_scale)[row * (head_dim / group) + (32 * c) / group]);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // 8 nibbles of word j -> elements 8j .. 8j + 7
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = (float)((int)((w[j] >> (8 * e)) & 15u) - 8) * sc;
      const float b = (float)((int)((w[j] >> (8 * e + 4)) & 15u) - 8) * sc;
      const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
      o[e] = *reinterpret_cast<const uint32_t*>(&p);
    }
    __stcs(dst + j, make_uint4(o[0], o[1], o[2], o[3]));  // streaming: the rows are not read back here
  }
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_gather_kv_f4(uint16_t* k_out, uint16_t* v_out, int64_t n_out, const uint8_t* k_data,
                                const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                const int32_t* page_table, const int32_t* seq_lens, const int64_t* out_start,
                                int32_t n_seq, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                int32_t max_pages_per_seq, int64_t num_pages, int32_t v_group,
                                int32_t* device_status, qkv_stream_t stream) {
  if (n_seq == 0) return QKV_OK;
  if (!k_out || !v_out || !k_data || !k_scale || !v_data || !v_scale || !page_table || !seq_lens || !out_start)
    return QKV_EINVAL;
  if (n_seq < 0 || n_seq > 65535 || n_out < 0 || kv_heads < 1 || head_dim < 32 || head_dim > 256 ||
      head_dim % 32 || block_size < 1 || max_pages_per_seq < 1 || num_pages < 1 ||
      (v_group != 32 && v_group != head_dim))
    return QKV_EINVAL;
  if (((uintptr_t)k_out | (uintptr_t)v_out | (uintptr_t)k_data | (uintptr_t)v_data) & 15) return QKV_EINVAL;
  if (((uintptr_t)k_scale | (uintptr_t)v_scale) & 1) return QKV_EINVAL;
  const int64_t threads = (int64_t)max_pages_per_seq * block_size * kv_heads * 2 * (head_dim / 32);
  const int64_t blocks = (threads + 255) / 256;
  if (threads > 0x7fffffff) return QKV_EUNSUPPORTED;
  __half* ks = reinterpret_cast<__half*>(const_cast<uint16_t*>(k_scale));
  __half* vs = reinterpret_cast<__half*>(const_cast<uint16_t*>(v_scale));
  int mp = max_pages_per_seq, kvh = kv_heads, hd = head_dim, bs = block_size, vg = v_group;
  void* args[] = {&k_data, &ks, &v_data, &vs, &page_table, &mp, &seq_lens, &out_start, &kvh, &hd, &bs,
                  &num_pages, &vg, &n_out, &k_out, &v_out, &device_status};
  if (launch_pdl((const void*)gather_kv_f4_kernel, dim3((unsigned)blocks, (unsigned)n_seq), dim3(256), 0, stream,
                 args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}
