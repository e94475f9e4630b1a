// lse_merge.cu -- log2-sum-exp fold of partial attention results (sm_100a).
//
// Source: FreeToken issue #568 "Serving ...'s 1M-token window on one 24 GB
// card", proposed solution item 2 (partials folded by log2-sum-exp); the
// v2 paged attention "reduce" step of mistral.rs PR "YaRN rope scaling, 4-bit
// F4 packed KV cache, ...", section 2.
//
// Per row: M = max_i lse2_i, w_i = 2^(lse2_i - M), out = sum_i w_i o_i /
// sum_i w_i, lse2 = M + log2 sum_i w_i. One CTA per (row, 64-dim chunk):
// 8 groups of 16 lanes split the parts, each lane carries 4 dims.
#include <math.h>

#include "common.cuh"

namespace qkv {

constexpr int MERGE_THREADS = 128;
constexpr int MERGE_GROUPS = MERGE_THREADS / 16;
constexpr int MERGE_DIMS = 64;

__global__ void __launch_bounds__(MERGE_THREADS) lse_merge_kernel(const float* __restrict__ o_parts,
                                                                  const float* __restrict__ lse2_parts,
                                                                  int n_parts, int rows, int head_dim,
                                                                  __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse2_out) {
  pdl_wait();
  pdl_release();
  __shared__ float red[MERGE_THREADS / 32];
  __shared__ float4 part[MERGE_GROUPS][16];
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
  for (int w = 1; w < MERGE_THREADS / 32; ++w) M = fmaxf(M, red[w]);
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
  for (int w = 0; w < MERGE_THREADS / 32; ++w) W += red[w];

  // weighted sum of this CTA's 64 dims
  const int grp = tid >> 4, l16 = tid & 15;
  const int d = blockIdx.y * MERGE_DIMS + 4 * l16;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (M != -INFINITY && d < head_dim)
    for (int i = grp; i < n_parts; i += MERGE_GROUPS) {
      const float l = lse2_parts[(size_t)i * rows + row];
      if (l == -INFINITY) continue;
      const float w = exp2f(l - M);
      const float4 x = *reinterpret_cast<const float4*>(o_parts + ((size_t)i * rows + row) * head_dim + d);
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
    }
  part[grp][l16] = acc;
  __syncthreads();
  if (grp == 0 && d < head_dim) {
    float4 s = part[0][l16];
#pragma unroll
    for (int g = 1; g < MERGE_GROUPS; ++g) {
      const float4 x = part[g][l16];
      s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    __nv_bfloat162 lo = __floats2bfloat162_rn(s.x * inv, s.y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(s.z * inv, s.w * inv);
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + (size_t)row * head_dim + d);
    dst[0] = lo;
    dst[1] = hi;
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
