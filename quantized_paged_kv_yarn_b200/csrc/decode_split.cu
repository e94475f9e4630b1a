// decode_split.cu -- split pass of paged GQA decode attention over the F4
// cache, and the one-call decode attention (split pass + log2-sum-exp merge).
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2
// (v1/v2 paged attention that dequantises F4 cells inline; v2 partitions the
// context and reduces the partitions); FreeToken issue #568 "Serving ...'s
// 1M-token window on one 24 GB card", proposed solution item 2 (partials
// folded by log2-sum-exp); ignis docs "context-and-speculation" (64-token KV
// pages; lanes sharing one pool).
//
// Design (B200, sm_100a). The step streams bytes: 288 bytes of packed K/V and
// scales per token and KV head feed 2 x 4 x 256 multiply-adds. One CTA owns
// (split, sequence, KV head) so the G query heads of the group share every
// dequantised page; 4 warps, 3 CTAs per SM (168 registers per thread).
//  * 64-token stages (one 64-token page, or 2/4 pages of 32/16 tokens) fill a
//    3-slot shared-memory ring: the packed K and V rows by 2-D TMA with the
//    128-byte swizzle, their fp16 scales by 1-D bulk copies, all completing
//    on one mbarrier per slot. Warp w issues the stages R = w (mod 4), so the
//    issue work is spread evenly and no warp paces the others; a slot is
//    refilled once all four warps have released it.
//  * Each warp takes 16 tokens of a stage. ldmatrix delivers the packed
//    nibbles already in mma-fragment order (plain for K, transposed for V).
//    Q K^T and P V run on the tensor cores as m16n8k16 fp16 MMAs with fp32
//    accumulation. K nibbles enter the MMA raw, as fp16 subnormals
//    (n * 2^-24 in bits 0-3, n * 2^-20 in bits 4-7, both exact): q carries
//    16 q on the low-nibble positions and each 32-dim cell's MMA chain starts
//    from -8 * 2^-20 * sum(q over the cell), so the chain yields
//    2^-20 * sum((n - 8) q) with one AND per fp16 pair. V nibbles enter the
//    same way; there the -8 offset is one extra MMA per tile, the sum over
//    tokens of p * v_scale per (cell, head), subtracted in the epilogue.
//    Each cell chain of K is scaled by that token's cell scale in fp32; the
//    per-cell V scale is folded into the probabilities (the B operand) of
//    that cell.
//  * The running max / sum live in registers (base-2 exponent); the four
//    warps are combined through shared memory and the CTA writes one fp32
//    partial and its lse2 per query head. The merge kernel folds splits.
// Dequantised tiles never touch shared memory: staging fp16 tiles for
// tcgen05 would need ~4x the shared-memory bandwidth of the packed bytes.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace qkv {

namespace split {
constexpr int D = 256;               // head_dim
constexpr int CELLS = D / 32;        // 8 cells of 32 values per row
constexpr int ROW_BYTES = D / 2;     // 128 packed bytes per token
constexpr int SROW_BYTES = CELLS * 2;  // 16 bytes of fp16 scales per token
constexpr int STAGE_TOK = 64;
constexpr int NS = 3;                // ring depth
constexpr int CWARPS = 4;            // warps; each takes 16 tokens of a stage
constexpr int THREADS = CWARPS * 32;
constexpr int TR_STRIDE = 20;        // padded row of the score transpose buffer

struct __align__(1024) Smem {
  uint8_t k[NS][STAGE_TOK * ROW_BYTES];  // 8 KiB each, 1024-aligned (128B swizzle atom)
  uint8_t v[NS][STAGE_TOK * ROW_BYTES];
  uint8_t ks[NS][STAGE_TOK * SROW_BYTES];
  uint8_t vs[NS][STAGE_TOK * SROW_BYTES];
  float tr[CWARPS][8][TR_STRIDE];
  uint4 qfrag[CELLS][32];  // per cell and lane: the 4 fp16x2 B registers of both k-steps
  float qbias[CELLS][8];   // per cell and head: -8 * 2^-20 * sum of the cell's q (accumulator start)
  float wm[CWARPS][8];
  float wl[CWARPS][8];
  unsigned long long mask[NS];
  uint64_t full[NS];
  uint64_t empty[NS];
  int abort_flag;
  int issued;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;  // + alignment slack

struct Params {
  float* o_parts;
  float* lse2_parts;
  const uint16_t* q;
  const uint16_t* k_scale;
  const uint16_t* v_scale;
  const int32_t* page_table;
  const int32_t* seq_lens;
  int32_t* status;
  int64_t num_pages;
  int n_seq, q_heads, kv_heads, max_pages, max_splits, num_splits, target;
  float score_scale;  // softmax_scale * log2(e)
};
}  // namespace split

using namespace split;

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// D = A * B + C with C given separately (no copy of C into D first).
__device__ __forceinline__ void mma_f16_c(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1, float c0, float c1, float c2, float c3) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

// 2^x for the softmax weights (hardware approximation, subnormal results flushed to 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float half_at(const uint4& v, int i) {
  const uint32_t w = (i < 2) ? v.x : (i < 4) ? v.y : (i < 6) ? v.z : v.w;
  const unsigned short b = (i & 1) ? (unsigned short)(w >> 16) : (unsigned short)(w & 0xffff);
  return __half2float(__ushort_as_half(b));
}

// Context length of a sequence, clamped to what its page-table row holds.
__device__ __forceinline__ int seq_len_of(const Params& p, int s, int block, bool report) {
  int L = p.seq_lens[s];
  const int cap = p.max_pages * block;
  if (L < 0 || L > cap) {
    if (report) flag(p.status, QKV_DEV_BAD_SEQLEN);
    L = L < 0 ? 0 : cap;
  }
  return L;
}

// Split plan. Fixed: min(num_splits, max_splits) splits per sequence.
// Automatic: pages are cut into pieces of about total pages / target, so the
// grid holds at most `target` busy CTAs per KV head whatever the mix of
// lengths. Split i of a sequence with n pages covers [i*n/S, (i+1)*n/S).
__device__ long long splits_for(const Params& p, int block, long long P) {
  long long total = 0;
  for (int s = 0; s < p.n_seq; ++s) total += ((seq_len_of(p, s, block, false) + block - 1) / block + P - 1) / P;
  return total;
}

__device__ void plan(const Params& p, int seq, int split, int block, int& S, int& pg0, int& pg1, int& L) {
  L = seq_len_of(p, seq, block, split == 0 && blockIdx.z == 0);
  const int n = (L + block - 1) / block;
  if (p.num_splits > 0) {
    S = min(p.num_splits, p.max_splits);
  } else {
    // Pieces of P pages with sum_s ceil(n_s / P) <= target, so the busy CTAs
    // fit the resident slots in one wave.
    long long T = 0, nmax = 1;
    for (int s = 0; s < p.n_seq; ++s) {
      const long long ns = (seq_len_of(p, s, block, false) + block - 1) / block;
      T += ns;
      nmax = max(nmax, ns);
    }
    long long P;
    if (p.target <= p.n_seq) {
      P = nmax;  // one split per sequence
    } else {
      P = max(1LL, (T + p.target - 1) / p.target);
      for (int k = 0; k < 4 && splits_for(p, block, P) > p.target; ++k) ++P;
      if (splits_for(p, block, P) > p.target) P = max(P, (T + p.target - p.n_seq - 1) / (p.target - p.n_seq));
    }
    S = (int)min((long long)p.max_splits, max(1LL, (n + P - 1) / P));
  }
  pg0 = (int)((long long)split * n / S);
  pg1 = (int)((long long)(split + 1) * n / S);
}

template <int BLOCK, int G>
__global__ void __launch_bounds__(THREADS, 3)
    paged_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                              const Params p) {
  static_assert(STAGE_TOK % BLOCK == 0, "pages must tile a stage");
  static_assert(G >= 1 && G <= 8, "one n8 MMA tile holds the query group");
  constexpr int PPS = STAGE_TOK / BLOCK;  // pages per stage

  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  pdl_wait();
  pdl_release();
  const int split = blockIdx.x, seq = blockIdx.y, kvh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = p.n_seq * p.q_heads;
  const int row0 = seq * p.q_heads + kvh * G;  // first query-head row of this group
  float* lse_out = p.lse2_parts + (size_t)split * rows + row0;

  int S, pg0, pg1, L;
  plan(p, seq, split, BLOCK, S, pg0, pg1, L);
  if (split >= S) {  // unused slot of the plan
    if (threadIdx.x < G) lse_out[threadIdx.x] = -INFINITY;
    return;
  }
  const int t_begin = pg0 * BLOCK;
  const int t_end = min(pg1 * BLOCK, L);
  const int n_it = t_end > t_begin ? (t_end - t_begin + STAGE_TOK - 1) / STAGE_TOK : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], CWARPS);
    }
    sm.abort_flag = 0;
    sm.issued = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ copy issue
  // Stage `it` holds tokens t_begin + 64 it ... +63, i.e. 64 / BLOCK pages,
  // each as four copies (K rows, V rows by TMA with the 128-byte swizzle; K
  // and V scales by bulk copy). Warp w issues the stages R = w (mod 4), so
  // the issue work is spread evenly over the warps; lane j of warp w keeps
  // the page ids of the j-th next of those stages (32 per refresh, the next
  // 32 prefetched), so no copy waits on a page-table load.
  const uint64_t pol = policy_evict_first();
  const int32_t* pt = p.page_table + (size_t)seq * p.max_pages + pg0;
  const int npg = pg1 - pg0;
  volatile int* abort_flag = &sm.abort_flag;
  int id_cur[PPS], id_nxt[PPS];
  int id_base = 0;  // index (R / CWARPS) of the stage held by lane 0
  auto load_ids = [&](int base, int (&dst)[PPS]) {
    const int R = (base + lane) * CWARPS + warp;
#pragma unroll
    for (int k = 0; k < PPS; ++k) {
      const int pi = R * PPS + k;
      dst[k] = pi < npg ? pt[pi] : -1;
    }
  };
  load_ids(0, id_cur);
  load_ids(32, id_nxt);
  // called by all lanes of warp R % CWARPS, with R increasing
  auto issue = [&](int R) {
    const int st = R % NS;
    const int j = R / CWARPS;
    if (j >= id_base + 32) {
      id_base += 32;
#pragma unroll
      for (int k = 0; k < PPS; ++k) id_cur[k] = id_nxt[k];
      load_ids(id_base + 32, id_nxt);
    }
    int phys[PPS];
#pragma unroll
    for (int k = 0; k < PPS; ++k) phys[k] = __shfl_sync(FULL_MASK, id_cur[k], (j - id_base) & 31);
    if (lane != 0) return;
    const int tok0 = t_begin + R * STAGE_TOK;
    unsigned long long mask = 0;
    uint32_t bytes = 0;
#pragma unroll
    for (int k = 0; k < PPS; ++k) {
      const int tk = tok0 + k * BLOCK;
      if (tk >= t_end) {
        phys[k] = -1;
        continue;
      }
      if (phys[k] < 0 || (int64_t)phys[k] >= p.num_pages) {
        flag(p.status, QKV_DEV_BAD_PAGE);
        phys[k] = -1;
        continue;
      }
      const int nv = min(BLOCK, t_end - tk);
      const unsigned long long bits = nv >= 64 ? ~0ull : ((1ull << nv) - 1ull);
      mask |= bits << (k * BLOCK);
      bytes += 2u * BLOCK * (ROW_BYTES + SROW_BYTES);
    }
    sm.mask[st] = mask;
    mbar_arrive_expect_tx(&sm.full[st], bytes);
#pragma unroll
    for (int k = 0; k < PPS; ++k) {
      if (phys[k] < 0) continue;
      const int row = (phys[k] * p.kv_heads + kvh) * BLOCK;
      tma_load_2d(&sm.k[st][k * BLOCK * ROW_BYTES], &tm_k, &sm.full[st], 0, row, pol);
      tma_load_2d(&sm.v[st][k * BLOCK * ROW_BYTES], &tm_v, &sm.full[st], 0, row, pol);
      bulk_load(&sm.ks[st][k * BLOCK * SROW_BYTES], p.k_scale + (size_t)row * CELLS, BLOCK * SROW_BYTES,
                &sm.full[st], pol);
      bulk_load(&sm.vs[st][k * BLOCK * SROW_BYTES], p.v_scale + (size_t)row * CELLS, BLOCK * SROW_BYTES,
                &sm.full[st], pol);
    }
    atomicMax(&sm.issued, R + 1);
  };
  if (warp < min(NS, n_it)) issue(warp);  // stages 0 .. NS-1

  // ------------------------------------------------------------ consumers
  const int g = lane >> 2, t = lane & 3;

  // q as the B operand (k = head_dim slice, n = query head). Within each
  // 32-dim cell the k index is permuted to match the nibble order the
  // unpack produces: k-step ks, fragment register r, half i <-> dim
  // 8t + 2ks + r + 4i.
  uint32_t qb[CELLS][2][2];  // built here, kept in shared memory
  float score_scale = p.score_scale;
  {
    float qf[CELLS][8];
    float qmax = 0.f;
#pragma unroll
    for (int c = 0; c < CELLS; ++c) {
      if (g < G) {
        const uint4 raw = *reinterpret_cast<const uint4*>(p.q + (size_t)(row0 + g) * D + 32 * c + 8 * t);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          qf[c][2 * i] = __uint_as_float(w[i] << 16);
          qf[c][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qf[c][i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) qmax = fmaxf(qmax, fabsf(qf[c][i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(FULL_MASK, qmax, o));
    // q enters the MMA as fp16 with an exact power-of-two prescale: the
    // low-nibble positions take 16 q (their K values are n * 2^-24), the
    // high-nibble positions q (K values n * 2^-20), so every product is
    // 2^-20 * n * q; 16 * max|q| stays below 2^15.
    const int qexp = (int)((__float_as_uint(qmax) >> 23) & 0xff) - 127;
    const int shift = qexp >= 11 ? qexp - 10 : 0;
    score_scale = ldexpf(score_scale, shift + 20);
#pragma unroll
    for (int c = 0; c < CELLS; ++c) {
      float qs = 0.f;  // sum of this lane's 8 dims of the cell, as the MMA sees them
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const __half2 lo = __floats2half2_rn(ldexpf(qf[c][2 * ks], -shift), ldexpf(qf[c][2 * ks + 4], -shift));
        const __half2 hi = __floats2half2_rn(ldexpf(qf[c][2 * ks + 1], -shift), ldexpf(qf[c][2 * ks + 5], -shift));
        const float2 lf = __half22float2(lo), hf = __half22float2(hi);
        qs += (lf.x + lf.y) + (hf.x + hf.y);
        qb[c][ks][0] = h2_as_u32(__hmul2(lo, u32_as_h2(0x4C004C00u)));  // x16, exact
        qb[c][ks][1] = h2_as_u32(hi);
      }
      qs += __shfl_xor_sync(FULL_MASK, qs, 1);
      qs += __shfl_xor_sync(FULL_MASK, qs, 2);
      if (warp == 0 && t == 0) sm.qbias[c][g] = (g < G) ? -8.0f * ldexpf(qs, -20) : 0.f;
    }
    if (warp == 0)
#pragma unroll
      for (int c = 0; c < CELLS; ++c) sm.qfrag[c][lane] = make_uint4(qb[c][0][0], qb[c][0][1], qb[c][1][0], qb[c][1][1]);
  }
  __syncthreads();

  float acc[CELLS][2][4];
#pragma unroll
  for (int c = 0; c < CELLS; ++c)
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[c][k][i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  // vsum[j] = running sum over tokens of p(token, head 2t+j) * v_scale(token, cell g)
  float vsum[2] = {0.f, 0.f};

  // ldmatrix row owned by this lane: matrix mi = lane / 8 covers tokens
  // 8 * (mi & 1) .. +7 of the warp's 16 and cell 2 * cp + (mi >> 1).
  const uint32_t ld_row = (uint32_t)((((lane >> 3) & 1) * 8 + (lane & 7)) * ROW_BYTES);
  const int sw = lane & 7;  // 128B swizzle: chunk index ^= row index mod 8
  const int co = lane >> 4;
  uint32_t ld_off[CELLS / 2];  // this lane's ldmatrix address offset for cell pair cp
#pragma unroll
  for (int cp = 0; cp < CELLS / 2; ++cp) ld_off[cp] = ld_row + ((uint32_t)((2 * cp + co) ^ sw) << 4);
  float(*tr)[TR_STRIDE] = sm.tr[warp];
  bool aborted = false;

  for (int it = 0; it < n_it; ++it) {
    const int st = it % NS;
    if (!aborted && !mbar_wait_bounded(&sm.full[st], (it / NS) & 1)) {
      flag(p.status, QKV_DEV_TIMEOUT);
      *abort_flag = 1;
    }
    // warp-uniform, so the .aligned ldmatrix / mma below see a converged warp
    aborted = __any_sync(FULL_MASK, aborted || (*abort_flag != 0));
    const uint32_t tmask = aborted ? 0u : (uint32_t)((sm.mask[st] >> (16 * warp)) & 0xffffu);
    if (tmask != 0u) {
      const uint32_t kbase = smem_u32(&sm.k[st][warp * 16 * ROW_BYTES]);
      const uint32_t vbase = smem_u32(&sm.v[st][warp * 16 * ROW_BYTES]);
      const uint8_t* ksb = &sm.ks[st][warp * 16 * SROW_BYTES];
      const uint8_t* vsb = &sm.vs[st][warp * 16 * SROW_BYTES];
      const bool partial = tmask != 0xffffu;

      const uint4 skA = lds128(ksb + g * SROW_BYTES);
      const uint4 skB = lds128(ksb + (g + 8) * SROW_BYTES);
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
      const uint32_t ka[4] = {skA.x, skA.y, skA.z, skA.w}, kb[4] = {skB.x, skB.y, skB.z, skB.w};
#pragma unroll
      for (int grp = 0; grp < 2; ++grp) {
        uint32_t kw[2][4];
        ldsm_x4(kbase + ld_off[2 * grp], kw[0]);
        ldsm_x4(kbase + ld_off[2 * grp + 1], kw[1]);
        float d[4][4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = 4 * grp + cc;
          const uint4 qv = sm.qfrag[c][lane];
          const float2 bias = *reinterpret_cast<const float2*>(&sm.qbias[c][2 * t]);
          const uint32_t wa = kw[cc >> 1][2 * (cc & 1)], wb = kw[cc >> 1][2 * (cc & 1) + 1];
          const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
          // raw nibbles as fp16 subnormals: n * 2^-24 (bits 0-3), n * 2^-20 (bits 4-7)
          mma_f16_c(d[cc], wa & 0x000F000Fu, wb & 0x000F000Fu, wa & 0x00F000F0u, wb & 0x00F000F0u, qv.x, qv.y,
                    bias.x, bias.y, bias.x, bias.y);
          mma_f16(d[cc], wa8 & 0x000F000Fu, wb8 & 0x000F000Fu, wa8 & 0x00F000F0u, wb8 & 0x00F000F0u, qv.z, qv.w);
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const float2 fa = __half22float2(u32_as_h2(ka[2 * grp + c2])), fb = __half22float2(u32_as_h2(kb[2 * grp + c2]));
          s0 = fmaf(fa.x, d[2 * c2][0], s0);
          s1 = fmaf(fa.x, d[2 * c2][1], s1);
          s2 = fmaf(fb.x, d[2 * c2][2], s2);
          s3 = fmaf(fb.x, d[2 * c2][3], s3);
          s0 = fmaf(fa.y, d[2 * c2 + 1][0], s0);
          s1 = fmaf(fa.y, d[2 * c2 + 1][1], s1);
          s2 = fmaf(fb.y, d[2 * c2 + 1][2], s2);
          s3 = fmaf(fb.y, d[2 * c2 + 1][3], s3);
        }
      }
      uint4 sv0 = lds128(vsb + (2 * t) * SROW_BYTES);
      uint4 sv1 = lds128(vsb + (2 * t + 1) * SROW_BYTES);
      uint4 sv2 = lds128(vsb + (2 * t + 8) * SROW_BYTES);
      uint4 sv3 = lds128(vsb + (2 * t + 9) * SROW_BYTES);
      s0 *= score_scale; s1 *= score_scale; s2 *= score_scale; s3 *= score_scale;
      if (partial) {
        if (!((tmask >> g) & 1u)) s0 = s1 = -INFINITY;
        if (!((tmask >> (g + 8)) & 1u)) s2 = s3 = -INFINITY;
        // the weights of absent tokens are exactly 0; make their scales 0 too
        // (a stale slot may hold any bit pattern)
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        if (!((tmask >> (2 * t)) & 1u)) sv0 = z4;
        if (!((tmask >> (2 * t + 1)) & 1u)) sv1 = z4;
        if (!((tmask >> (2 * t + 8)) & 1u)) sv2 = z4;
        if (!((tmask >> (2 * t + 9)) & 1u)) sv3 = z4;
      }

      // ---- transpose to the PV B-operand layout: head g, tokens 2t, 2t+1, 2t+8, 2t+9
      __syncwarp();
      if (2 * t < G) {
        tr[2 * t][g] = s0;
        tr[2 * t][g + 8] = s2;
        if (2 * t + 1 < G) {
          tr[2 * t + 1][g] = s1;
          tr[2 * t + 1][g + 8] = s3;
        }
      }
      __syncwarp();
      float sc[4];
      if (g < G) {
        const float2 a = *reinterpret_cast<const float2*>(&tr[g][2 * t]);
        const float2 b = *reinterpret_cast<const float2*>(&tr[g][2 * t + 8]);
        sc[0] = a.x; sc[1] = a.y; sc[2] = b.x; sc[3] = b.y;
      } else {
        sc[0] = sc[1] = sc[2] = sc[3] = -INFINITY;
      }

      // ---- online softmax in base 2 (per head g; lanes of one g agree)
      float mt = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
      mt = fmaxf(mt, __shfl_xor_sync(FULL_MASK, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(FULL_MASK, mt, 2));
      const float m_new = fmaxf(m_run, mt);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (g < G) ? ex2(m_run - m_use) : 1.f;
      float pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pr[i] = ex2(sc[i] - m_use);
      l_run = l_run * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
      m_run = m_new;
      const float al0 = __shfl_sync(FULL_MASK, alpha, (8 * t) & 31);
      const float al1 = __shfl_sync(FULL_MASK, alpha, (8 * t + 4) & 31);
      if (__any_sync(FULL_MASK, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < CELLS; ++c)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            acc[c][k][0] *= al0; acc[c][k][1] *= al1;
            acc[c][k][2] *= al0; acc[c][k][3] *= al1;
          }
        vsum[0] *= al0;
        vsum[1] *= al1;
      }

      // ---- P V with the V scale folded into P per cell (packed fp16). The V
      // nibbles enter raw, as fp16 subnormals (n * 2^-24 on MMA rows 0-7,
      // n * 2^-20 on rows 8-15); the -8 offset is accounted for once per
      // tile by vsum += S_v^T P (cell x head), applied in the epilogue.
      const __half2 p01 = __floats2half2_rn(pr[0], pr[1]), p23 = __floats2half2_rn(pr[2], pr[3]);
      const uint32_t s0w[4] = {sv0.x, sv0.y, sv0.z, sv0.w}, s1w[4] = {sv1.x, sv1.y, sv1.z, sv1.w};
      const uint32_t s2w[4] = {sv2.x, sv2.y, sv2.z, sv2.w}, s3w[4] = {sv3.x, sv3.y, sv3.z, sv3.w};
      {
        // A = the tile's V scales transposed: row = cell g, k = tokens 2t, 2t+1 (+8)
        uint32_t st0, st1;
        ldsm_x2_trans(smem_u32(vsb) + (uint32_t)((lane & 15) * SROW_BYTES), st0, st1);
        if (partial) {  // absent tokens: a stale slot may hold any bit pattern
          st0 &= (((tmask >> (2 * t)) & 1u) ? 0x0000ffffu : 0u) | (((tmask >> (2 * t + 1)) & 1u) ? 0xffff0000u : 0u);
          st1 &= (((tmask >> (2 * t + 8)) & 1u) ? 0x0000ffffu : 0u) | (((tmask >> (2 * t + 9)) & 1u) ? 0xffff0000u : 0u);
        }
        float dd[4];
        mma_f16_c(dd, st0, 0u, st1, 0u, h2_as_u32(p01), h2_as_u32(p23), vsum[0], vsum[1], 0.f, 0.f);
        vsum[0] = dd[0];
        vsum[1] = dd[1];
      }
      uint32_t vw[2][4];
#pragma unroll
      for (int c = 0; c < CELLS; ++c) {
        if ((c & 1) == 0) ldsm_x4_trans(vbase + ld_off[c >> 1], vw[(c >> 1) & 1]);
        const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;
        const uint32_t b01 = h2_as_u32(__hmul2(p01, u32_as_h2(__byte_perm(s0w[c >> 1], s1w[c >> 1], sel))));
        const uint32_t b23 = h2_as_u32(__hmul2(p23, u32_as_h2(__byte_perm(s2w[c >> 1], s3w[c >> 1], sel))));
        const uint32_t za = vw[(c >> 1) & 1][2 * (c & 1)], zb = vw[(c >> 1) & 1][2 * (c & 1) + 1];
        const uint32_t za8 = za >> 8, zb8 = zb >> 8;
        mma_f16(acc[c][0], za & 0x000F000Fu, za & 0x00F000F0u, zb & 0x000F000Fu, zb & 0x00F000F0u, b01, b23);
        mma_f16(acc[c][1], za8 & 0x000F000Fu, za8 & 0x00F000F0u, zb8 & 0x000F000Fu, zb8 & 0x00F000F0u, b01, b23);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);
    // The slot of the previous iteration (all warps have normally left it by
    // now) is refilled NS - 1 iterations ahead of its use, by its own warp.
    if (it >= 1 && it - 1 + NS < n_it && ((it - 1 + NS) % CWARPS) == warp) {
      const int pv = it - 1;
      int go = 1;
      if (lane == 0) {
        if (*abort_flag) {
          go = 0;
        } else if (!mbar_wait_bounded(&sm.empty[pv % NS], (pv / NS) & 1)) {
          flag(p.status, QKV_DEV_TIMEOUT);
          *abort_flag = 1;
          go = 0;
        }
      }
      if (__shfl_sync(FULL_MASK, go, 0)) issue(pv + NS);
    }
  }

  // ------------------------------------------------------------ combine the 4 warps
  l_run += __shfl_xor_sync(FULL_MASK, l_run, 1);
  l_run += __shfl_xor_sync(FULL_MASK, l_run, 2);
  if (t == 0 && g < G) {
    sm.wm[warp][g] = m_run;
    sm.wl[warp][g] = l_run;
  }
  __syncthreads();
  if (*abort_flag) {
    // Leave only after every copy issued here has landed.
    if (threadIdx.x == 0) {
      const int issued = sm.issued;
      for (int it = max(0, issued - NS); it < issued; ++it)
        if (!mbar_wait_bounded(&sm.full[it % NS], (it / NS) & 1)) flag(p.status, QKV_DEV_TIMEOUT);
    }
    if (threadIdx.x < G) lse_out[threadIdx.x] = -INFINITY;
    return;
  }
  // Each warp scales its accumulator to the CTA-wide max and parks it in
  // the (now idle) K ring: slab[warp][head][dim].
  float* slab = reinterpret_cast<float*>(&sm.k[0][0]);
  float fw[2] = {0.f, 0.f};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int h = 2 * t + j;
    if (h < G) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < CWARPS; ++w) M = fmaxf(M, sm.wm[w][h]);
      fw[j] = (M == -INFINITY) ? 0.f : exp2f(sm.wm[warp][h] - M);
    }
  }
  // Undo the subnormal encoding of V: rows 0-7 carry 2^-24 * sum(n p s),
  // rows 8-15 2^-20 * sum(n p s); the -8 offset is 8 * sum(p s) per cell.
#pragma unroll
  for (int c = 0; c < CELLS; ++c) {
    const float b0 = 8.f * __shfl_sync(FULL_MASK, vsum[0], 4 * c + t);
    const float b1 = 8.f * __shfl_sync(FULL_MASK, vsum[1], 4 * c + t);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      acc[c][k][0] = fmaf(acc[c][k][0], 16777216.f, -b0);
      acc[c][k][1] = fmaf(acc[c][k][1], 16777216.f, -b1);
      acc[c][k][2] = fmaf(acc[c][k][2], 1048576.f, -b0);
      acc[c][k][3] = fmaf(acc[c][k][3], 1048576.f, -b1);
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int h = 2 * t + j;
    if (h < G) {
      float* dst = slab + ((size_t)warp * 8 + h) * D;
#pragma unroll
      for (int c = 0; c < CELLS; ++c) {
        const float4 o = make_float4(fw[j] * acc[c][0][j], fw[j] * acc[c][0][j + 2], fw[j] * acc[c][1][j],
                                     fw[j] * acc[c][1][j + 2]);
        *reinterpret_cast<float4*>(dst + 32 * c + 4 * g) = o;
      }
    }
  }
  __syncthreads();
  // Sum the warps, normalise, write the partial of this split.
  const int tid = threadIdx.x;  // 0 .. 127
  for (int e = tid; e < G * (D / 4); e += CWARPS * 32) {
    const int h = e / (D / 4), d4 = e % (D / 4);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < CWARPS; ++w) M = fmaxf(M, sm.wm[w][h]);
    float Lsum = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < CWARPS; ++w) {
      const float f = (M == -INFINITY) ? 0.f : exp2f(sm.wm[w][h] - M);
      Lsum += f * sm.wl[w][h];
      const float4 x = *reinterpret_cast<const float4*>(slab + ((size_t)w * 8 + h) * D + 4 * d4);
      o.x += x.x; o.y += x.y; o.z += x.z; o.w += x.w;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    o.x *= inv; o.y *= inv; o.z *= inv; o.w *= inv;
    *reinterpret_cast<float4*>(p.o_parts + ((size_t)split * rows + row0 + h) * D + 4 * d4) = o;
    if (d4 == 0) lse_out[h] = Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
  }
}

}  // namespace qkv

// ======================================================================= host side

using namespace qkv;

namespace {

using EncodeTiled = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(ptr);
  });
  return fn;
}

// 2-D view [rows][128 bytes] of a packed cache, boxes of `block` rows,
// 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, int block) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)ROW_BYTES, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ROW_BYTES};
  const cuuint32_t box[2] = {(cuuint32_t)ROW_BYTES, (cuuint32_t)block};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BLOCK, int G>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&paged_decode_split_kernel<BLOCK, G>);
}

const void* pick_kernel(int block, int G) {
#define QKV_PICK(B)                         \
  if (block == B) {                         \
    if (G == 1) return kernel_ptr<B, 1>();  \
    if (G == 2) return kernel_ptr<B, 2>();  \
    if (G == 4) return kernel_ptr<B, 4>();  \
    if (G == 8) return kernel_ptr<B, 8>();  \
  }
  QKV_PICK(16)
  QKV_PICK(32)
  QKV_PICK(64)
#undef QKV_PICK
  return nullptr;
}

constexpr int MAX_DEVICES = 64;

// Opt the kernel into its shared-memory size on the current device (once)
// and return its resident CTAs per SM.
int prepare(const void* fn, int block, int G) {
  static std::mutex mu;
  static int occ[MAX_DEVICES][3][4];  // 0 = not prepared
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return 0;
  const int bi = block == 16 ? 0 : block == 32 ? 1 : 2;
  const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  std::lock_guard<std::mutex> lock(mu);
  if (occ[dev][bi][gi] == 0) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES) != cudaSuccess)
      return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, THREADS, SMEM_BYTES) != cudaSuccess || n < 1)
      return 0;
    occ[dev][bi][gi] = n;
  }
  return occ[dev][bi][gi];
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

}  // namespace

extern "C" int32_t qkv_paged_decode_auto_splits(int32_t kv_heads, int32_t block_size) {
  if (kv_heads < 1) return 0;
  const void* fn = pick_kernel(block_size, 4);
  if (!fn) return 0;
  const int occ = prepare(fn, block_size, 4);
  const int sms = sm_count();
  if (occ < 1 || sms < 1) return 0;
  return (int32_t)std::max(1, occ * sms / kv_heads);
}

extern "C" size_t qkv_paged_decode_workspace_bytes(int32_t n_seq, int32_t q_heads, int32_t head_dim,
                                                   int32_t max_splits) {
  if (n_seq < 0 || q_heads < 0 || head_dim < 0 || max_splits < 0) return 0;
  const size_t rows = (size_t)n_seq * q_heads * max_splits;
  const size_t o = (rows * head_dim * 4 + 255) & ~size_t(255);
  const size_t l = (rows * 4 + 255) & ~size_t(255);
  return o + l;
}

extern "C" int qkv_paged_decode_split_f4(float* o_parts, float* lse2_parts, int32_t max_splits, const uint16_t* q,
                                         const uint8_t* k_data, const uint16_t* k_scale, const uint8_t* v_data,
                                         const uint16_t* v_scale, const int32_t* page_table,
                                         const int32_t* seq_lens, int32_t n_seq, int32_t q_heads,
                                         int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                         int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                         int32_t num_splits, int32_t* device_status, qkv_stream_t stream) {
  if (!o_parts || !lse2_parts || !q || !k_data || !k_scale || !v_data || !v_scale || !page_table || !seq_lens)
    return QKV_EINVAL;
  if (n_seq < 0 || q_heads < 1 || kv_heads < 1 || max_pages_per_seq < 1 || num_pages < 1 || max_splits < 1 ||
      num_splits < 0 || block_size < 1 || !(softmax_scale >= 0.f) || !isfinite(softmax_scale))
    return QKV_EINVAL;
  if (q_heads % kv_heads) return QKV_EINVAL;
  if (!aligned16(q) || !aligned16(k_data) || !aligned16(v_data) || !aligned16(k_scale) || !aligned16(v_scale) ||
      !aligned16(o_parts) || ((uintptr_t)lse2_parts & 3))
    return QKV_EINVAL;
  const int G = q_heads / kv_heads;
  if (head_dim != D) return QKV_EUNSUPPORTED;
  const void* fn = pick_kernel(block_size, G);
  if (!fn) return QKV_EUNSUPPORTED;
  const uint64_t cache_rows = (uint64_t)num_pages * kv_heads * block_size;
  if (cache_rows > 0x7fffffffull) return QKV_EUNSUPPORTED;  // TMA row coordinate is int32
  if ((int64_t)max_pages_per_seq * block_size > 0x7fffffffLL) return QKV_EUNSUPPORTED;
  if (max_splits > 65535 * 16 || n_seq > 65535 || kv_heads > 65535) return QKV_EUNSUPPORTED;
  if (n_seq == 0) return QKV_OK;

  const int occ = prepare(fn, block_size, G);
  const int sms = sm_count();
  if (occ < 1 || sms < 1) return QKV_ECUDA;

  CUtensorMap tm_k, tm_v;
  if (!make_map(&tm_k, k_data, cache_rows, block_size) || !make_map(&tm_v, v_data, cache_rows, block_size))
    return QKV_ECUDA;

  Params p;
  p.o_parts = o_parts;
  p.lse2_parts = lse2_parts;
  p.q = q;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.page_table = page_table;
  p.seq_lens = seq_lens;
  p.status = device_status;
  p.num_pages = num_pages;
  p.n_seq = n_seq;
  p.q_heads = q_heads;
  p.kv_heads = kv_heads;
  p.max_pages = max_pages_per_seq;
  p.max_splits = max_splits;
  p.num_splits = num_splits;
  p.target = std::max(1, occ * sms / kv_heads);
  const float sc = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf((float)head_dim);
  p.score_scale = sc * 1.4426950408889634f;

  // Slots past the plan's split count still get lse2 = -inf: the grid
  // covers every slot the merge reads.
  dim3 grid((unsigned)max_splits, (unsigned)n_seq, (unsigned)kv_heads);
  void* args[] = {(void*)&tm_k, (void*)&tm_v, (void*)&p};
  if (launch_pdl(fn, grid, dim3(THREADS), SMEM_BYTES, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" int qkv_paged_decode_attn_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                                        const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                        const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                        int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                        int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                        int32_t num_splits, int32_t max_splits, void* workspace,
                                        size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream) {
  if (!out || !workspace) return QKV_EINVAL;
  if (((uintptr_t)workspace & 255) || max_splits < 1 || n_seq < 0 || q_heads < 1) return QKV_EINVAL;
  if (workspace_bytes < qkv_paged_decode_workspace_bytes(n_seq, q_heads, head_dim, max_splits)) return QKV_EINVAL;
  if (n_seq == 0) return QKV_OK;
  const size_t rows = (size_t)n_seq * q_heads;
  float* o_parts = reinterpret_cast<float*>(workspace);
  float* lse_parts =
      reinterpret_cast<float*>((char*)workspace + ((rows * max_splits * head_dim * 4 + 255) & ~size_t(255)));
  int rc = qkv_paged_decode_split_f4(o_parts, lse_parts, max_splits, q, k_data, k_scale, v_data, v_scale,
                                     page_table, seq_lens, n_seq, q_heads, kv_heads, head_dim, block_size,
                                     max_pages_per_seq, num_pages, softmax_scale, num_splits, device_status, stream);
  if (rc != QKV_OK) return rc;
  return qkv_lse_merge(o_parts, lse_parts, max_splits, (int32_t)rows, head_dim, out, lse2_out, stream);
}
