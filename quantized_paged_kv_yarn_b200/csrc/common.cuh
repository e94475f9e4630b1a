// common.cuh -- device helpers shared by the kernels of the decode hot path
// (sm_100a): shared-memory addressing, mbarriers with bounded waits, TMA and
// bulk copies, ldmatrix and warp-level MMA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qkv.h"

#define QKV_LAUNCH_CHECK()                                 \
  do {                                                     \
    if (cudaPeekAtLastError() != cudaSuccess) {            \
      (void)cudaGetLastError();                            \
      return QKV_ECUDA;                                    \
    }                                                      \
  } while (0)

namespace qkv {

constexpr unsigned FULL_MASK = 0xffffffffu;

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

// Programmatic dependent launch. Every kernel of the library is launched
// with programmatic stream serialization allowed, so it may be scheduled
// while its predecessor in the stream is still running. On every path, and
// before it reads anything a kernel ahead of it may write, it calls
// pdl_wait(), which returns once the predecessor grid has completed and its
// writes are visible (so a grid's completion implies its predecessors').
// pdl_release() lets the successor be scheduled: kernels call it at their
// start, except those that write the K/V cache (the F4 writes and the
// staging of host pages) or the rotary table, which leave it to their
// completion. The split pass of decode attention reads the page table, the
// sequence lengths, cache pages and (the decode step's) positions, slots
// and rotary table before it waits; that is safe because no kernel that
// released its successor early writes them.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch with programmatic stream serialization allowed (see pdl_wait).
inline cudaError_t launch_pdl(const void* kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, kernel, args);
}

__device__ __forceinline__ void flag(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// NEOX rotation of the pair (x0, x1) = (x_j, x_{j+rot/2}) by (c, s), float,
// with a fixed rounding order so every kernel produces the same bits.
__device__ __forceinline__ float rot_first(float x0, float x1, float c, float s) {
  return __fmaf_rn(x0, c, -__fmul_rn(x1, s));
}
__device__ __forceinline__ float rot_second(float x0, float x1, float c, float s) {
  return __fmaf_rn(x1, c, __fmul_rn(x0, s));
}

// Row helpers for one K or V head row of a token spread over a warp: lane l
// holds elements 8 l .. 8 l + 7 (lanes past head_dim / 8 hold zeros). All
// 32 lanes must call them.

// NEOX rotation of dims [0, rot) in place, rounded to bf16 as qkv_rope_apply
// rounds its output; the partner of dim j < rot / 2 is j + rot / 2, which sits
// rot / 16 lanes away (rot is a multiple of 16). cos_row / sin_row: the
// position's table row.
// The table values lane l needs for the rotation of its 8 elements (as
// rope_row_bf16_cs uses them); lanes past rot / 8 load nothing.
__device__ __forceinline__ void rope_load_cs(int lane, int rot, const float* cos_row, const float* sin_row,
                                             float (&c)[8], float (&s)[8]) {
  const int half = rot / 2;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = lane * 8 + i;
    c[i] = s[i] = 0.f;
    if (j < rot) {
      const int jj = j < half ? j : j - half;
      c[i] = cos_row[jj];
      s[i] = sin_row[jj];
    }
  }
}

// rope_row_bf16 with the table values already loaded (rope_load_cs).
__device__ __forceinline__ void rope_row_bf16_cs(float (&x)[8], int lane, int rot, const float (&c)[8],
                                                 const float (&s)[8]) {
  const int half = rot / 2, dl = half / 8;
  float y[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float other = __shfl_sync(0xffffffffu, x[i], lane < dl ? lane + dl : lane - dl);
    y[i] = x[i];
    const int j = lane * 8 + i;
    if (j < rot)
      y[i] = __bfloat162float(__float2bfloat16_rn(j < half ? rot_first(x[i], other, c[i], s[i])
                                                           : rot_second(other, x[i], c[i], s[i])));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = y[i];
}

__device__ __forceinline__ void rope_row_bf16(float (&x)[8], int lane, int rot, const float* cos_row,
                                              const float* sin_row) {
  float c[8], s[8];
  rope_load_cs(lane, rot, cos_row, sin_row, c, s);
  rope_row_bf16_cs(x, lane, rot, c, s);
}

// F4 quantise-write of the row (as qkv_kv_write_f4): scale = fp16(amax / 7)
// per `group` values (32, or head_dim: one scale for the row), codes
// rint(x / scale) clamped to [-8, 7] + 8, low nibble first. data_row: the
// row's head_dim / 2 packed bytes; scale_row: its head_dim / group scales.
// (Both divisions are IEEE; the results are exact, as argued in kv_write.cu.)
__device__ __forceinline__ void f4_write_row(const float (&x)[8], int lane, int head_dim, int group,
                                             uint8_t* data_row, __half* scale_row) {
  const bool active = lane * 8 < head_dim;
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
  // lanes per scale group: 4 for a 32-value cell; the whole warp for a group
  // of head_dim values (lanes past head_dim / 8 hold amax 0)
  const int gl = group == 32 ? 4 : 32;
  for (int o = 1; o < gl; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
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
  reinterpret_cast<uint32_t*>(data_row)[lane] = word;
  if ((lane & (gl - 1)) == 0) scale_row[lane / gl] = sh;
}

// Row of 8 bf16 per lane as float (zeros past head_dim).
__device__ __forceinline__ void load_row8(const uint16_t* row, int lane, int head_dim, float (&x)[8]) {
  if (lane * 8 < head_dim) {
    const uint4 raw = *reinterpret_cast<const uint4*>(row + lane * 8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = 0.f;
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// WAIT_LIMIT_NS. Returns false when the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 255u) == 0 && globaltimer() - t0 > WAIT_LIMIT_NS) return false;
  }
}

// ---------------------------------------------------------------- copies

// 2-D tiled TMA load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// 1-D bulk copy global -> shared (no multicast); both addresses 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- ldmatrix / mma

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// D += A * B, m16n8k16, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

}  // namespace qkv
