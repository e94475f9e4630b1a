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

// One CTA per (row, 64-dim chunk); 8 warps split the parts (warp w takes
// parts w, w + 8, ...). A warp loads the lse2 of up to 32 of its parts (one
// per lane) together with the 64-dim rows (2 dims per lane) of the first 8 of
// them, before their weights are known: the rows of parts without weight are
// selected away, never multiplied, so whatever they hold is harmless. With
// up to 8 parts per warp (64 per row) the fold costs one global-latency
// round. The warps' (max, weight sum, weighted sum) are combined in shared
// memory. (Eight warps rather than sixteen: the merge's CTAs then hold fewer
// of the SMs that the next split launch's CTAs wait for; 0.607 against
// 0.612 ms per 16-layer decode step at 131,072 tokens, the same at 262,144.)
constexpr int MERGE_WARPS = 8;
constexpr int MERGE_THREADS = MERGE_WARPS * 32;
constexpr int MERGE_DIMS = 64;
constexpr int MERGE_BATCH = 8;  // part rows a lane has in flight at once

__global__ void __launch_bounds__(MERGE_THREADS) lse_merge_kernel(const float* __restrict__ o_parts,
                                                                  const float* __restrict__ lse2_parts,
                                                                  int n_parts, int rows, int head_dim,
                                                                  __nv_bfloat16* __restrict__ out,
                                                                  float* __restrict__ lse2_out) {
  pdl_release();
  pdl_wait();
  __shared__ float wm[MERGE_WARPS], wsum[MERGE_WARPS];
  __shared__ float2 wacc[MERGE_WARPS][32];
  const int row = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = blockIdx.y * MERGE_DIMS + 2 * lane;
  const bool dim_ok = d < head_dim;

  // running (max, weight sum, weighted sum) of this warp's parts
  float m = -INFINITY, ws = 0.f;
  float2 acc = make_float2(0.f, 0.f);
  for (int base = warp; base < n_parts; base += MERGE_WARPS * 32) {
    // lane j holds part base + 16 j of this round
    const int my = base + MERGE_WARPS * lane;
    const int cnt = min(32, (n_parts - base + MERGE_WARPS - 1) / MERGE_WARPS);
    auto load_rows = [&](int j0, float2 (&x)[MERGE_BATCH]) {
#pragma unroll
      for (int u = 0; u < MERGE_BATCH; ++u) {
        const int j = j0 + u;
        x[u] = make_float2(0.f, 0.f);
        if (j < cnt && dim_ok)
          x[u] = *reinterpret_cast<const float2*>(o_parts + ((size_t)(base + MERGE_WARPS * j) * rows + row) * head_dim + d);
      }
    };
    float2 x[MERGE_BATCH];
    load_rows(0, x);
    const float l = my < n_parts ? lse2_parts[(size_t)my * rows + row] : -INFINITY;
    float mr = l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mr = fmaxf(mr, __shfl_xor_sync(FULL_MASK, mr, o));
    if (mr == -INFINITY) continue;  // nothing in this round
    const float mn = fmaxf(m, mr);
    const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    acc.x *= alpha;
    acc.y *= alpha;
    ws *= alpha;
    m = mn;
    const float wt = (l == -INFINITY) ? 0.f : exp2f(l - m);
    float wsr = wt;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wsr += __shfl_xor_sync(FULL_MASK, wsr, o);
    ws += wsr;
    for (int j0 = 0; j0 < cnt; j0 += MERGE_BATCH) {
      if (j0 > 0) load_rows(j0, x);
#pragma unroll
      for (int u = 0; u < MERGE_BATCH; ++u) {
        const float w = __shfl_sync(FULL_MASK, wt, (j0 + u) & 31);
        if (j0 + u < cnt && w != 0.f) {
          acc.x = fmaf(w, x[u].x, acc.x);
          acc.y = fmaf(w, x[u].y, acc.y);
        }
      }
    }
  }
  if (lane == 0) {
    wm[warp] = m;
    wsum[warp] = ws;
  }
  wacc[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < MERGE_WARPS; ++w) M = fmaxf(M, wm[w]);
    float W = 0.f;
    float2 o = make_float2(0.f, 0.f);
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < MERGE_WARPS; ++w) {
        const float f = (wm[w] == -INFINITY) ? 0.f : exp2f(wm[w] - M);
        W = fmaf(f, wsum[w], W);
        const float2 a = wacc[w][lane];
        o.x = fmaf(f, a.x, o.x);
        o.y = fmaf(f, a.y, o.y);
      }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    if (dim_ok)
      *reinterpret_cast<__nv_bfloat162*>(out + (size_t)row * head_dim + d) = __floats2bfloat162_rn(o.x * inv, o.y * inv);
    if (lane == 0 && blockIdx.y == 0 && lse2_out) lse2_out[row] = W > 0.f ? M + log2f(W) : -INFINITY;
  }
}

// Few parts per row (the chunked prefill's context split, a short decode
// plan): one warp per (row, 64-dim chunk), eight to a CTA, each lane holding
// the lse2 of part `lane` and the rows of every part for its 2 dims, all
// loaded at once; no shared memory and no block barrier. (The 2048-query
// prefill chunk with its 4-part split: 10.77 against 11.05 ms with the
// many-part kernel, whose idle warps then outnumber the busy ones.)
constexpr int MERGE_SMALL_PARTS = 8;

__global__ void __launch_bounds__(256) lse_merge_small_kernel(const float* __restrict__ o_parts,
                                                              const float* __restrict__ lse2_parts, int n_parts,
                                                              int rows, int head_dim, int chunks,
                                                              __nv_bfloat16* __restrict__ out,
                                                              float* __restrict__ lse2_out) {
  pdl_release();
  pdl_wait();
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);  // (row, chunk)
  const int lane = threadIdx.x & 31;
  if (item >= rows * chunks) return;
  const int row = item / chunks, chunk = item - row * chunks;
  const int d = chunk * MERGE_DIMS + 2 * lane;
  const bool dim_ok = d < head_dim;
  float2 x[MERGE_SMALL_PARTS];
#pragma unroll
  for (int j = 0; j < MERGE_SMALL_PARTS; ++j) {
    x[j] = make_float2(0.f, 0.f);
    if (j < n_parts && dim_ok)
      x[j] = *reinterpret_cast<const float2*>(o_parts + ((size_t)j * rows + row) * head_dim + d);
  }
  const float l = lane < n_parts ? lse2_parts[(size_t)lane * rows + row] : -INFINITY;
  float M = l;
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, o));  // lanes 0-7 hold the parts
  M = __shfl_sync(FULL_MASK, M, 0);
  const float wt = (l == -INFINITY) ? 0.f : exp2f(l - M);
  float W = 0.f;
  float2 o = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < MERGE_SMALL_PARTS; ++j) {
    const float w = __shfl_sync(FULL_MASK, wt, j);
    W += w;
    if (j < n_parts && w != 0.f) {  // unweighted rows are never multiplied
      o.x = fmaf(w, x[j].x, o.x);
      o.y = fmaf(w, x[j].y, o.y);
    }
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
  if (dim_ok)
    *reinterpret_cast<__nv_bfloat162*>(out + (size_t)row * head_dim + d) = __floats2bfloat162_rn(o.x * inv, o.y * inv);
  if (lane == 0 && chunk == 0 && lse2_out) lse2_out[row] = W > 0.f ? M + log2f(W) : -INFINITY;
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_lse_merge(const float* o_parts, const float* lse2_parts, int32_t n_parts, int32_t rows,
                             int32_t head_dim, uint16_t* out, float* lse2_out, qkv_stream_t stream) {
  if (!o_parts || !lse2_parts || !out) return QKV_EINVAL;
  if (n_parts < 1 || rows < 0 || head_dim < 4 || head_dim % 4 || head_dim > 1024) return QKV_EINVAL;
  if (((uintptr_t)o_parts & 15) || ((uintptr_t)lse2_parts & 3) || ((uintptr_t)out & 3) ||
      ((uintptr_t)lse2_out & 3))
    return QKV_EINVAL;
  if (rows == 0) return QKV_OK;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(out);
  int np = n_parts, nr = rows, hd = head_dim;
  if (n_parts <= MERGE_SMALL_PARTS) {
    int chunks = (head_dim + MERGE_DIMS - 1) / MERGE_DIMS;
    const long long items = (long long)rows * chunks;
    if (items > 0x7fffffffLL) return QKV_EUNSUPPORTED;
    void* sargs[] = {&o_parts, &lse2_parts, &np, &nr, &hd, &chunks, &o, &lse2_out};
    if (launch_pdl((const void*)lse_merge_small_kernel, dim3((unsigned)((items + 7) / 8)), dim3(256), 0, stream,
                   sargs) != cudaSuccess) {
      (void)cudaGetLastError();
      return QKV_ECUDA;
    }
    return QKV_OK;
  }
  dim3 grid((unsigned)rows, (unsigned)((head_dim + MERGE_DIMS - 1) / MERGE_DIMS));
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
