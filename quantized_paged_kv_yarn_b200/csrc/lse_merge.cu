// lse_merge.cu -- log2-sum-exp fold of partial attention results (sm_100a).
//
// Source: FreeToken issue #568 "Serving ...'s 1M-token window on one 24 GB
// card", proposed solution item 2 (partials folded by log2-sum-exp); the
// v2 paged attention "reduce" step of mistral.rs PR "YaRN rope scaling, 4-bit
// F4 packed KV cache, ...", section 2.
//
// Per row: M = max_i lse2_i, w_i = 2^(lse2_i - M), out = sum_i w_i o_i /
// sum_i w_i, lse2 = M + log2 sum_i w_i.
#include <math.h>

#include "common.cuh"

namespace qkv {

// One CTA per (row, 128-dim chunk). 16 warps split the parts (warp w takes
// parts w, w + 16, ...); each lane carries 4 dims, so a warp covers the
// chunk. A thread issues the loads of all its parts before using them.
constexpr int MERGE_WARPS = 16;
constexpr int MERGE_THREADS = MERGE_WARPS * 32;
constexpr int MERGE_DIMS = 128;
constexpr int MERGE_UNROLL = 8;  // parts per warp in flight

__global__ void __launch_bounds__(MERGE_THREADS) lse_merge_kernel(const float* __restrict__ o_parts,
                                                                  const float* __restrict__ lse2_parts,
                                                                  int n_parts, int rows, int head_dim,
                                                                  __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse2_out) {
  pdl_wait();
  pdl_release();
  __shared__ float red[MERGE_WARPS];
  __shared__ float4 part[MERGE_WARPS][32];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // M and the weight sum over all parts
  float m = -INFINITY;
  for (int i = tid; i < n_parts; i += MERGE_THREADS) m = fmaxf(m, lse2_parts[(size_t)i * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL_MASK, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < MERGE_WARPS; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float ws = 0.f;
  if (M != -INFINITY)
    for (int i = tid; i < n_parts; i += MERGE_THREADS) {
      const float l = lse2_parts[(size_t)i * rows + row];
      if (l != -INFINITY) ws += exp2f(l - M);
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ws += __shfl_xor_sync(FULL_MASK, ws, o);
  if (lane == 0) red[warp] = ws;
  __syncthreads();
  float W = 0.f;
#pragma unroll
  for (int w = 0; w < MERGE_WARPS; ++w) W += red[w];

  // weighted sum of this CTA's dims, MERGE_UNROLL parts per warp at a time
  const int d = blockIdx.y * MERGE_DIMS + 4 * lane;
  const bool dim_ok = d < head_dim;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY && dim_ok)
    for (int base = warp; base < n_parts; base += MERGE_WARPS * MERGE_UNROLL) {
      float lw[MERGE_UNROLL];
      float4 x[MERGE_UNROLL];
#pragma unroll
      for (int u = 0; u < MERGE_UNROLL; ++u) {
        const int i = base + u * MERGE_WARPS;
        lw[u] = i < n_parts ? lse2_parts[(size_t)i * rows + row] : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < MERGE_UNROLL; ++u) {
        const int i = base + u * MERGE_WARPS;
        x[u] = (lw[u] != -INFINITY) ? *reinterpret_cast<const float4*>(o_parts + ((size_t)i * rows + row) * head_dim + d)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < MERGE_UNROLL; ++u) {
        const float w = (lw[u] != -INFINITY) ? exp2f(lw[u] - M) : 0.f;
        acc.x = fmaf(w, x[u].x, acc.x);
        acc.y = fmaf(w, x[u].y, acc.y);
        acc.z = fmaf(w, x[u].z, acc.z);
        acc.w = fmaf(w, x[u].w, acc.w);
      }
    }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && dim_ok) {
    float4 s = part[0][lane];
#pragma unroll
    for (int w = 1; w < MERGE_WARPS; ++w) {
      const float4 x = part[w][lane];
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + (size_t)row * head_dim + d);
    dst[0] = __floats2bfloat162_rn(s.x * inv, s.y * inv);
    dst[1] = __floats2bfloat162_rn(s.z * inv, s.w * inv);
  }
  if (tid == 0 && blockIdx.y == 0 && lse2_out) lse2_out[row] = W > 0.f ? M + log2f(W) : -INFINITY;
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_lse_merge(const float* o_parts, const float* lse2_parts, int32_t n_parts, int32_t rows,
                             int32_t head_dim, uint16_t* out, float* lse2_out, qkv_stream_t stream) {
  if (!o_parts || !lse2_parts || !out) return QKV_EINVAL;
  if (n_parts < 1 || rows < 0 || head_dim < 4 || head_dim % 4 || head_dim > 1024) return QKV_EINVAL;
  if (((uintptr_t)o_parts & 15) || ((uintptr_t)lse2_parts & 3) || ((uintptr_t)out & 7) ||
      ((uintptr_t)lse2_out & 3))
    return QKV_EINVAL;
  if (rows == 0) return QKV_OK;
  dim3 grid((unsigned)rows, (unsigned)((head_dim + MERGE_DIMS - 1) / MERGE_DIMS));
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  int np = n_parts, nr = rows, hd = head_dim;
  void* args[] = {&o_parts, &lse2_parts, &np, &nr, &hd, &o, &lse2_out};
  if (launch_pdl((const void*)lse_merge_kernel, grid, dim3(MERGE_THREADS), 0, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" const char* qkv_status_string(int status) {
  switch (status) {
    case QKV_OK: return "ok";
    case QKV_EINVAL: return "invalid argument";
    case QKV_EUNSUPPORTED: return "unsupported shape";
    case QKV_ECUDA: return "CUDA error";
    default: return "unknown status";
  }
}
