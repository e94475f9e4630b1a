#pragma once
// decode_split.cuh -- the split pass of paged GQA decode attention over the F4
// cache (device code), for head_dim 256 and 128.
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2
// (v1/v2 paged attention that dequantises F4 cells inline; v2 partitions the
// context and reduces the partitions); FreeToken issue #568 "Serving ...'s
// 1M-token window on one 24 GB card", proposed solution item 2 (partials
// folded by log2-sum-exp); ignis docs "context-and-speculation" (64-token KV
// pages; lanes sharing one pool).
//
// Design (B200, sm_100a). The step streams bytes: per token and KV head,
// 288 (head_dim 256) or 144 (128) bytes of packed K/V and scales feed
// 2 x G x head_dim multiply-adds. One CTA owns (split, sequence, KV head) so
// the G query heads of the group share every page it reads: one 512-thread
// CTA per SM, made of four independent 4-warp groups that share the split's
// 64-token stages (the first INIT of each round-robin, then claimed from a
// shared-memory counter, so the four finish within about a stage of each
// other); their partials are folded in shared memory at the end.
//  * Staging, per group: the packed K rows and their fp16 scales fill a
//    2-slot K ring, the V rows and scales a 3-slot V ring (V of a stage is
//    read last): rows by 2-D TMA with the swizzle of the row width (128-byte
//    rows: 128B, 64-byte rows: 64B), scales by 1-D bulk copies, L2
//    evict-first, each half of a stage on its own mbarrier. Local stage j + 2
//    is issued at the group barrier of local stage j by warp (j + 2) mod 4,
//    which claimed it (and read its page ids) four stages earlier.
//  * Q K^T: warp w scores tokens 16w .. 16w + 15 of the stage. ldmatrix
//    delivers the packed nibbles in mma-fragment order and they enter an
//    m16n8k16 fp16 MMA (fp32 accumulate) raw, as fp16 subnormals (n * 2^-24
//    in bits 0-3, n * 2^-20 in bits 4-7): q carries 16 q on the low-nibble
//    positions and the -8 code offset is the chain's start value, -8 * 2^-20
//    * sum(q over the cell). One MMA covers two cells: its 8 columns are
//    (query head, cell parity), so each lane ends with both cells of one
//    head and scales them by their own per-token cell scales in fp32.
//  * Softmax: base-2 scores against one running max m per head shared by the
//    group, probabilities 2^(x - m - SLACK). A stage whose scores all stay
//    below m + SLACK (after the first stages, nearly all) needs one group
//    barrier: the warps write their probabilities (fp16) to shared memory and
//    the barrier, which also ORs a "new max" flag, publishes them. Otherwise
//    the warps exchange tile maxima, rescale and rewrite.
//  * P V: warp w owns the dims of cells 2w, 2w + 1 (head_dim 128: cell w)
//    over all 64 tokens of the stage: V^T (ldmatrix.trans, nibbles as fp16
//    subnormals) is the A operand, P times the token's V cell scale (one
//    packed fp16 multiply) the B operand. The -8 offset is sum_t p * v_scale
//    per (cell, head): one extra MMA per warp and stage over the warp's own
//    16 tokens (summed across the group's warps at the end), or, when one B
//    operand serves all of a warp's cells (one V scale per token, or
//    head_dim 128), an MMA with an all-ones A per 16 tokens.
//  * The loop is software-pipelined: an iteration multiplies stage i into
//    the accumulators and scores stage i + 1 in one block.
//  * The CTA writes one fp32 partial per query head and its lse2; the merge
//    kernel folds the splits.
// Dequantised tiles never touch shared memory: staging fp16 tiles for
// tcgen05 would need ~4x the shared-memory bandwidth of the packed bytes.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "common.cuh"

namespace qkv {

namespace split {
// Per head_dim D (256 or 128): 32-value cells per row, cell pairs (one MMA
// chain each), packed bytes and fp16 scale bytes per token row, cells per
// warp in P V.
template <int D>
struct Geo {
  static constexpr int CELLS = D / 32;
  static constexpr int PAIRS = CELLS / 2;
  static constexpr int ROW_BYTES = D / 2;
  static constexpr int SROW_BYTES = CELLS * 2;
  static constexpr int CPW = CELLS / 4;
};
constexpr int STAGE_TOK = 64;
constexpr int NSK = 2;                 // K ring depth
constexpr int NSV = 3;                 // V ring depth (V of a stage is read last)
constexpr int GWARPS = 4;              // warps of a group; a group processes whole stages
constexpr int GROUPS = 4;              // groups per CTA, sharing the split's stages
constexpr int GTHREADS = GWARPS * 32;
constexpr int THREADS = GROUPS * GTHREADS;
constexpr int INIT = 6;                // a group's first local stages, assigned without claims
constexpr int PROW = STAGE_TOK + 8;    // padded probability row (fp16): conflict-free B loads
constexpr uint32_t LO4 = 0x000F000Fu;  // nibble of bits 0-3 of each 16-bit half
constexpr uint32_t HI4 = 0x00F000F0u;  // nibble of bits 4-7 of each 16-bit half
// The running max of a head moves only when a score exceeds it by more than
// SLACK (base-2 units); probabilities are taken against m + SLACK, so they
// stay <= 1 and the fp16 product p * v_scale cannot overflow.
constexpr float SLACK = 2.0f;

// Query-head quads: G <= 4 heads fit one MMA tile of (head, cell parity)
// columns; G = 8 takes two.
template <int G>
struct Cfg {
  static constexpr int HQ = (G + 3) / 4;
};

// One group's rings, probabilities and bookkeeping.
template <int D>
struct __align__(1024) GroupSmem {
  uint8_t k[NSK][STAGE_TOK * Geo<D>::ROW_BYTES];  // 8 (4) KiB each, 1024-aligned (swizzle atom)
  uint8_t v[NSV][STAGE_TOK * Geo<D>::ROW_BYTES];
  uint8_t ks[NSK][STAGE_TOK * Geo<D>::SROW_BYTES];
  uint8_t vs[NSV][STAGE_TOK * Geo<D>::SROW_BYTES];
  uint16_t prob[2][8][PROW];  // fp16 probabilities [stage parity][query head][token]
  float tmax[GWARPS][8];
  float wl[GWARPS][8];
  unsigned long long mask[NSK];  // tokens present in the stage of each K slot
  uint64_t kfull[NSK];
  uint64_t vfull[NSV];
  int n_local;  // the group's stage count, once a claim ran past the split
  int issued;   // local stages issued so far
};

template <int HQ, int D>
struct __align__(1024) Smem {
  GroupSmem<D> grp[GROUPS];
  uint4 qfrag[HQ][Geo<D>::PAIRS][2][32];  // per lane: the B registers of the 4 MMAs of a cell pair
  float4 qbias[HQ][Geo<D>::PAIRS][4];     // per lane t: chain start of columns 2t, 2t+1 (twice, rows g and g+8)
  float gm[GROUPS][8];            // per group and head: exponent reference of its sums
  float gl[GROUPS][8];            // per group and head: softmax sum
  int next;                       // next stage of the split to claim
  int abort_flag;
};
template <int HQ, int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<HQ, D>) + 1024;  // + alignment slack
}

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
// The decode step's inputs (qkv_decode_step_f4): q is unrotated; the kernel
// rotates it and writes the step's new K (rotated) and V into the cache
// first. Only the fused instances take them: a larger parameter block made
// ptxas compile the plain kernel's loop 1.2 us slower.
struct StepFields {
  int rot, v_group;
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int64_t* positions;
  const int64_t* slots;
  const float* cos_tab;
  const float* sin_tab;
  int64_t tab_start, tab_len;
  uint8_t* k_data_w;
  uint8_t* v_data_w;
  __half* k_scale_w;
  __half* v_scale_w;
};
template <bool FUSE>
struct KParams : Params {};
template <>
struct KParams<true> : Params {
  StepFields st;
};
}  // namespace split

using namespace split;

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint2 lds64(const void* p) { return *reinterpret_cast<const uint2*>(p); }
__device__ __forceinline__ uint32_t lds32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }

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

// Named barrier `id` over one group's GTHREADS threads that also returns the
// OR of `pred` over them.
__device__ __forceinline__ bool bar_red_or(uint32_t id, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "n"(GTHREADS)
      : "memory");
  return out != 0;
}

__device__ __forceinline__ void bar_sync(uint32_t id) { asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(GTHREADS) : "memory"); }

// Wait for phase `parity` of a copy barrier. False when the CTA is aborting
// (another warp set the flag) or the wait limit ran out (then this sets it).
__device__ __forceinline__ bool wait_copies(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                            int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > WAIT_LIMIT_NS) {
      flag(status, QKV_DEV_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
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

// ceil(a / b) for a >= 0, b > 0 (32-bit division: a few instructions)
__device__ __forceinline__ uint32_t cdiv(uint32_t a, uint32_t b) { return (a + b - 1) / b; }

// floor(a * b / c) for a, b >= 0, c > 0, in 32-bit arithmetic when a * b fits
__device__ __forceinline__ int muldiv(uint32_t a, uint32_t b, uint32_t c) {
  const unsigned long long ab = (unsigned long long)a * b;
  return (ab >> 32) == 0 ? (int)((uint32_t)ab / c) : (int)(ab / c);
}

// First page of split s (0 <= s <= S) of a sequence of n pages: S equal
// parts, except that splits 0 .. m-1 take d pages fewer each (the others
// share them). Those are the CTAs placed last (the grid runs splits in
// reverse order), which start a prologue's time after the rest when they
// get the SMs that the previous launch or its merge freed last. With
// P = n / S: bound(s) = s (P - d) for s <= m, and s P + d m (s - m) / (S - m)
// - d m for s >= m, rounded down (d <= P / 4 keeps it increasing).
__device__ inline int split_bound(uint32_t s, uint32_t n, uint32_t S, uint32_t m, uint32_t d) {
  if (m == 0 || d == 0) return muldiv(s, n, S);
  const long long den = (long long)S * (S - m);
  const long long num = s <= m ? ((long long)s * n - (long long)s * d * S) * (S - m)
                               : (long long)n * (S - m) * s - (long long)m * d * S * (S - s);
  return (int)(num / den);
}

// Split plan. Fixed: num_splits splits per sequence (the host refuses a
// count above max_splits).
// Automatic: pages are cut into pieces of about total pages / target, so the
// grid holds at most `target` busy CTAs per KV head whatever the mix of
// lengths. Split i covers pages [bound(i), bound(i + 1)) of its sequence:
// with S >= 8 splits the first ceil(S / 7) of them (the ones placed last)
// are `late_tok` tokens (at most a quarter split) shorter.
__device__ inline long long splits_for(const Params& p, int block, uint32_t P) {
  long long total = 0;
  for (int s = 0; s < p.n_seq; ++s) total += cdiv(cdiv((uint32_t)seq_len_of(p, s, block, false), block), P);
  return total;
}

__device__ inline void plan(const Params& p, int seq, int split, int block, int late_tok, int& S, int& pg0, int& pg1,
                            int& L) {
  L = seq_len_of(p, seq, block, split == 0 && blockIdx.x == 0);  // one report per sequence (KV head 0)
  const uint32_t n = cdiv((uint32_t)L, (uint32_t)block);
  if (p.num_splits > 0) {
    S = p.num_splits;
  } else {
    // Pieces of P pages with sum_s ceil(n_s / P) <= target, so the busy CTAs
    // fit the resident slots in one wave.
    long long T = 0;
    uint32_t nmax = 1;
    for (int s = 0; s < p.n_seq; ++s) {
      const uint32_t ns = cdiv((uint32_t)seq_len_of(p, s, block, false), (uint32_t)block);
      T += ns;
      nmax = max(nmax, ns);
    }
    uint32_t P;
    if (p.target <= p.n_seq) {
      P = nmax;  // one split per sequence
    } else {
      P = (uint32_t)max(1LL, (T + p.target - 1) / p.target);
      for (int k = 0; k < 4 && splits_for(p, block, P) > p.target; ++k) ++P;
      if (splits_for(p, block, P) > p.target)
        P = max(P, (uint32_t)((T + p.target - p.n_seq - 1) / (p.target - p.n_seq)));
    }
    S = (int)min((uint32_t)p.max_splits, max(1u, cdiv(n, P)));
  }
  const uint32_t m = S >= 8 ? ((uint32_t)S + 6) / 7 : 0;
  const uint32_t d = min((uint32_t)late_tok / (uint32_t)block, n / (uint32_t)S / 4);
  pg0 = split_bound((uint32_t)split, n, (uint32_t)S, m, d);
  pg1 = split_bound((uint32_t)split + 1, n, (uint32_t)S, m, d);
}

template <int D, int BLOCK, int G, bool VTOK, bool FUSE>
__global__ void __launch_bounds__(THREADS, 1)
    paged_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                              const KParams<FUSE> p) {
  static_assert(STAGE_TOK % BLOCK == 0, "pages must tile a stage");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "query heads per KV head");
  static_assert(D == 256 || D == 128, "head_dim");
  constexpr int CELLS = Geo<D>::CELLS, PAIRS = Geo<D>::PAIRS, ROW_BYTES = Geo<D>::ROW_BYTES;
  constexpr int SROW_BYTES = Geo<D>::SROW_BYTES, CPW = Geo<D>::CPW;
  constexpr int HQ = Cfg<G>::HQ;
  constexpr int PPS = STAGE_TOK / BLOCK;  // pages per stage
  // V scales: one per 32-value cell (16 bytes per token), or one per token
  constexpr int VSROW = VTOK ? 2 : SROW_BYTES;
  constexpr int VCELLS = VTOK ? 1 : CELLS;
  using SmemT = Smem<HQ, D>;

  // 1024-aligned (the 128-byte swizzle atom) by pointer arithmetic on the
  // shared array itself, so the compiler keeps every access through `sm` in
  // the shared window (32-bit addresses, shared loads) instead of generic
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SmemT& sm = *reinterpret_cast<SmemT*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));

  // Programmatic dependent launch. The kernel lets its successor launch at
  // once (the fused instance: once the CTA that writes the step's new token
  // has written it), and does everything that reads no output of the
  // kernels ahead of it before it waits for them: the split plan (sequence
  // lengths), the page ids and the first two stages' copies of every group.
  // Kernels ahead of it that let their successors start early write none of
  // these: the library's writers of the cache never do, and the fused
  // instance's own write is ordered before the copies of its stage below.
  if constexpr (!FUSE) pdl_release();
  // CTAs are placed in launch order as SMs free up, so the last ones land on
  // the SMs that the previous launch (or its merge) frees last and start
  // late. The grid runs the KV heads fastest and the splits in reverse
  // order: the late ones are the first splits of every KV head, which the
  // plan makes shorter, and not the sequence's last split, which holds the
  // new token's page (the decode step's write), nor the plan's unused slots
  // (which leave at once).
  const int kvh = blockIdx.x, split = (int)(gridDim.y - 1 - blockIdx.y), seq = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = warp / GWARPS, gw = warp % GWARPS;  // group, warp within the group
  const int g = lane >> 2, t = lane & 3;
  const int rows = p.n_seq * p.q_heads;
  const int row0 = seq * p.q_heads + kvh * G;  // first query-head row of this CTA
  float* lse_out = p.lse2_parts + (size_t)split * rows + row0;
  GroupSmem<D>& gs = sm.grp[grp];

  int S, pg0, pg1, L;
  // ~3 us of a late start at an SM's ~38 GB/s: 400 tokens of 288 bytes (head_dim 256)
  plan(p, seq, split, BLOCK, D == 256 ? 400 : 800, S, pg0, pg1, L);
  if (split >= S) {  // unused slot of the plan
    if constexpr (FUSE) pdl_release();
    pdl_wait();  // the workspace may still be read by the kernels ahead
    if (threadIdx.x < G) lse_out[threadIdx.x] = -INFINITY;
    return;
  }
  const int t_begin = pg0 * BLOCK;
  const int t_end = min(pg1 * BLOCK, L);
  const int n_it = t_end > t_begin ? (t_end - t_begin + STAGE_TOK - 1) / STAGE_TOK : 0;
  // Decode step: this CTA's split holds the sequence's last page, where the
  // step's new token goes; that page's stage (the split's last) is copied
  // only after the write.
  const int last_pg = (L - 1) / BLOCK;
  const bool writes_token = FUSE && L > 0 && last_pg >= pg0 && last_pg < pg1;
  if constexpr (FUSE) {
    if (!writes_token) pdl_release();
  }

  if (threadIdx.x == 0) {
    for (int q = 0; q < GROUPS; ++q) {
      for (int s = 0; s < NSK; ++s) mbar_init(&sm.grp[q].kfull[s], 1);
      for (int s = 0; s < NSV; ++s) mbar_init(&sm.grp[q].vfull[s], 1);
      // local stages j < INIT of group q are stages q + GROUPS j of the split
      const int valid = min(INIT, max(0, (n_it - q + GROUPS - 1) / GROUPS));
      sm.grp[q].n_local = valid < INIT ? valid : 0x7fffffff;
      sm.grp[q].issued = 0;
    }
    sm.next = GROUPS * INIT;
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  // probability rows of absent query heads (G < 8) are read as zeros
  for (int i = threadIdx.x % GTHREADS; i < (int)(sizeof(gs.prob) / 4); i += GTHREADS)
    reinterpret_cast<uint32_t*>(&gs.prob[0][0][0])[i] = 0u;
  __syncthreads();  // barriers initialised

  // ------------------------------------------------------------ copy issue
  // Stage R of the split holds tokens t_begin + 64 R ... + 63, i.e. 64 /
  // BLOCK pages. The four groups share the split's stages dynamically: a
  // group's local stage j is stage grp + 4 j for j < INIT, then whatever the
  // next claim on the CTA's counter returns, claimed in order, so a group
  // that runs faster takes more stages and all groups finish together. Local
  // stage j belongs to warp j % 4 of the group, which claims it four of its
  // stages ahead (with its page ids) and issues both halves of it (K rows and
  // scales on kfull[j % NSK], V on vfull[j % NSV]) at the group barrier of
  // local stage j - 2. The first claim past the split sets n_local, the
  // group's stage count.
  const uint64_t pol = policy_evict_first();
  const int32_t* pt = p.page_table + (size_t)seq * p.max_pages + pg0;
  const int npg = pg1 - pg0;
  const int full_stages = (t_end - t_begin) / STAGE_TOK;  // stages with all 64 tokens
  volatile int* abort_flag = &sm.abort_flag;
  volatile int* n_local = &gs.n_local;
  // the host keeps num_pages * kv_heads * block below 2^31
  const uint32_t num_pages32 = (uint32_t)p.num_pages;
  int held = n_it;  // stage of the split held for this warp's next local stage (>= n_it: none)
  int ids[PPS];
  // claim local stage j (all lanes of warp j % 4, j increasing by 4)
  auto claim = [&](int j) {
    int R;
    if (j < INIT) {
      R = grp + GROUPS * j;
    } else {
      R = 0;
      if (lane == 0) R = atomicAdd(&sm.next, 1);
      R = __shfl_sync(FULL_MASK, R, 0);
    }
    held = R;
    if (R >= n_it) {
      if (lane == 0 && j >= INIT) atomicMin(&gs.n_local, j);
      return;
    }
#pragma unroll
    for (int k = 0; k < PPS; ++k) {
      const int pi = R * PPS + k;
      ids[k] = pi < npg ? pt[pi] : -1;
    }
  };
  // issue local stage j and claim j + 4 (all lanes of warp j % 4)
  auto issue = [&](int j, bool copy) {
    const int R = held;
    int phys[PPS];
#pragma unroll
    for (int k = 0; k < PPS; ++k) phys[k] = ids[k];
    claim(j + GWARPS);
    if (R >= n_it || !copy || lane != 0) return;
    const int ks = j % NSK, vs = j % NSV;
    bool all_ok = R < full_stages;
#pragma unroll
    for (int k = 0; k < PPS; ++k) all_ok = all_ok && (uint32_t)phys[k] < num_pages32;
    unsigned long long mask = ~0ull;
    uint32_t npages = PPS;
    if (!all_ok) {  // the last, partial stage or an invalid page id
      const int tok0 = t_begin + R * STAGE_TOK;
      mask = 0;
      npages = 0;
#pragma unroll
      for (int k = 0; k < PPS; ++k) {
        const int tk = tok0 + k * BLOCK;
        if (tk >= t_end) {
          phys[k] = -1;
        } else if ((uint32_t)phys[k] >= num_pages32) {  // negative ids wrap to large
          flag(p.status, QKV_DEV_BAD_PAGE);
          phys[k] = -1;
        } else {
          const int nv = min(BLOCK, t_end - tk);
          const unsigned long long bits = nv >= 64 ? ~0ull : ((1ull << nv) - 1ull);
          mask |= bits << (k * BLOCK);
          ++npages;
        }
      }
    }
    gs.mask[ks] = mask;
    mbar_arrive_expect_tx(&gs.kfull[ks], npages * BLOCK * (ROW_BYTES + SROW_BYTES));
    mbar_arrive_expect_tx(&gs.vfull[vs], npages * BLOCK * (ROW_BYTES + VSROW));
#pragma unroll
    for (int k = 0; k < PPS; ++k) {
      if (phys[k] < 0) continue;
      const int row = (phys[k] * p.kv_heads + kvh) * BLOCK;
      tma_load_2d(&gs.k[ks][k * BLOCK * ROW_BYTES], &tm_k, &gs.kfull[ks], 0, row, pol);
      bulk_load(&gs.ks[ks][k * BLOCK * SROW_BYTES], p.k_scale + (size_t)row * CELLS, BLOCK * SROW_BYTES,
                &gs.kfull[ks], pol);
      tma_load_2d(&gs.v[vs][k * BLOCK * ROW_BYTES], &tm_v, &gs.vfull[vs], 0, row, pol);
      bulk_load(&gs.vs[vs][k * BLOCK * VSROW], p.v_scale + (size_t)row * VCELLS, BLOCK * VSROW, &gs.vfull[vs],
                pol);
    }
    atomicMax(&gs.issued, j + 1);
  };
  // Local stages 0 and 1 of every group now, before the wait (unless the
  // stage holds the page of the step's new token); stage j + 2 follows at
  // the group barrier of stage j.
  claim(gw);
  const bool first_copy = gw < 2;  // this warp issues a first stage
  const bool defer = writes_token && held == n_it - 1;
  if (first_copy && !defer) issue(gw, true);
  // Decode step: the step's position, rotary table values and slot are
  // metadata, read before the wait like the page table; q and the new k and
  // v are the step's activations, read after it.
  float rc[8] = {}, rs[8] = {};  // table values of this lane's 8 rotated dims
  bool pos_ok = false;
  int64_t slot = -1;
  if constexpr (FUSE) {
    const int half = p.st.rot / 2;
    const int64_t ti = p.st.positions[seq] - p.st.tab_start;
    pos_ok = ti >= 0 && ti < p.st.tab_len;
    if (!pos_ok && threadIdx.x == 0 && split == 0 && kvh == 0) flag(p.status, QKV_DEV_BAD_POSITION);
    if (pos_ok && (warp < G || warp == 8))
      rope_load_cs(lane, p.st.rot, p.st.cos_tab + ti * half, p.st.sin_tab + ti * half, rc, rs);
    if (writes_token && (warp == 8 || warp == 9)) slot = p.st.slots[seq];
  }
  pdl_wait();
  // Decode step: the CTA's query heads, rotated (bf16), in group 0's last V
  // slot, which is first written by the copy of its local stage 2, issued in
  // the main loop, after the q set-up has read them (8 KiB, 1024-aligned).
  uint16_t(*qrot)[D] = reinterpret_cast<uint16_t(*)[D]>(&sm.grp[0].v[NSV - 1][0]);
  static_assert(8 * D * 2 <= STAGE_TOK * ROW_BYTES, "qrot fits a V slot");
  if constexpr (FUSE) {
    // The decode step's rotary and F4 write inside this launch (as
    // qkv_rope_kv_write_f4 computes them): warp h < G rotates query head h
    // into shared memory; the CTA whose split holds the sequence's last
    // page writes the new token's K (rotated, warp 8) and V (warp 9) into the
    // cache before any of its copies starts.
    if (warp < G) {
      float x[8];
      load_row8(p.q + (size_t)(row0 + warp) * D, lane, D, x);
      if (pos_ok) rope_row_bf16_cs(x, lane, p.st.rot, rc, rs);
      uint4 o;  // the rotated values are bf16-exact
      o.x = (__float_as_uint(x[0]) >> 16) | (__float_as_uint(x[1]) & 0xffff0000u);
      o.y = (__float_as_uint(x[2]) >> 16) | (__float_as_uint(x[3]) & 0xffff0000u);
      o.z = (__float_as_uint(x[4]) >> 16) | (__float_as_uint(x[5]) & 0xffff0000u);
      o.w = (__float_as_uint(x[6]) >> 16) | (__float_as_uint(x[7]) & 0xffff0000u);
      if (8 * lane < D) *reinterpret_cast<uint4*>(&qrot[warp][8 * lane]) = o;
    }
    if (writes_token && (warp == 8 || warp == 9)) {
      const bool is_k = warp == 8;
      if (slot >= p.num_pages * BLOCK) {
        if (lane == 0 && is_k) flag(p.status, QKV_DEV_BAD_SLOT);
      } else if (slot >= 0) {
        float x[8];
        load_row8((is_k ? p.st.k_new : p.st.v_new) + ((size_t)seq * p.kv_heads + kvh) * D, lane, D, x);
        if (is_k && pos_ok) rope_row_bf16_cs(x, lane, p.st.rot, rc, rs);
        const int group = is_k ? 32 : p.st.v_group;
        const int64_t crw = ((slot / BLOCK) * p.kv_heads + kvh) * BLOCK + slot % BLOCK;
        f4_write_row(x, lane, D, group, (is_k ? p.st.k_data_w : p.st.v_data_w) + crw * ROW_BYTES,
                     (is_k ? p.st.k_scale_w : p.st.v_scale_w) + crw * (D / group));
        // the copies of this CTA (async proxy) read these bytes after the
        // barrier; the kernels after this one may read them once it lets
        // them start
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
      }
    }
  }
  __syncthreads();
  if (writes_token) pdl_release();
  if (first_copy && defer) issue(gw, true);

  // ------------------------------------------------------------ q as the B operand
  // Column n of the Q K^T tile is (query head n >> 1 of the quad, cell
  // parity n & 1). Lane (g, t) builds column g: head 4 hq + (g >> 1), cell
  // 2 pp + (g & 1), dims 8t .. 8t + 7 of that cell. The 4 MMAs of a pair
  // take the nibble variants v = 0..3 (dims 8t + v and 8t + 4 + v); rows 0-7
  // of the k index come from the even cell, rows 8-15 from the odd one.
  float score_scale = p.score_scale;
  {
    const int hl = g >> 1, par = g & 1;
    const bool col_ok = G >= 4 || hl < G;
    float qf[HQ][PAIRS][8];
    float qmax = 0.f;
#pragma unroll
    for (int hq = 0; hq < HQ; ++hq)
#pragma unroll
      for (int pp = 0; pp < PAIRS; ++pp) {
        if (col_ok) {
          uint4 raw;
          if constexpr (FUSE)  // rotated in shared memory
            raw = *reinterpret_cast<const uint4*>(&qrot[4 * hq + hl][32 * (2 * pp + par) + 8 * t]);
          else
            raw = *reinterpret_cast<const uint4*>(p.q + (size_t)(row0 + 4 * hq + hl) * D +
                                                  32 * (2 * pp + par) + 8 * t);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            qf[hq][pp][2 * i] = __uint_as_float(w[i] << 16);
            qf[hq][pp][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) qf[hq][pp][i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) qmax = fmaxf(qmax, fabsf(qf[hq][pp][i]));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(FULL_MASK, qmax, o));
    // q enters the MMA as fp16 with an exact power-of-two prescale: the
    // low-nibble positions take 16 q (their K values are n * 2^-24), the
    // high-nibble positions q (K values n * 2^-20), so every product is
    // 2^-20 * n * q; 16 * max|q| stays below 2^15.
    const int qexp = (int)((__float_as_uint(qmax) >> 23) & 0xff) - 127;
    const int shift = qexp >= 11 ? qexp - 10 : 0;
    // exact powers of two (shift <= 117): 2^-shift scales q, 2^(shift + 20) the scores
    const float down = __int_as_float((127 - shift) << 23);
    score_scale = score_scale * 1048576.f * __int_as_float((127 + shift) << 23);
#pragma unroll
    for (int hq = 0; hq < HQ; ++hq)
#pragma unroll
      for (int pp = 0; pp < PAIRS; ++pp) {
        uint32_t bv[4];
        float qs = 0.f;  // sum of this lane's 8 dims, as the MMA sees them
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const __half2 h = __floats2half2_rn(qf[hq][pp][v] * down, qf[hq][pp][v + 4] * down);
          const float2 f = __half22float2(h);
          qs += f.x + f.y;
          bv[v] = (v & 1) ? h2_as_u32(h) : h2_as_u32(__hmul2(h, u32_as_h2(0x4C004C00u)));  // x16, exact
        }
        uint32_t b0[4], b1[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          b0[v] = par ? 0u : bv[v];
          b1[v] = par ? bv[v] : 0u;
        }
        if (warp == 0) {
          sm.qfrag[hq][pp][0][lane] = make_uint4(b0[0], b1[0], b0[1], b1[1]);
          sm.qfrag[hq][pp][1][lane] = make_uint4(b0[2], b1[2], b0[3], b1[3]);
        }
        qs += __shfl_xor_sync(FULL_MASK, qs, 1);
        qs += __shfl_xor_sync(FULL_MASK, qs, 2);
        // column g starts its chain at -8 * 2^-20 * sum of the cell's q
        if (warp == 0 && t == 0) {
          float* b4 = reinterpret_cast<float*>(&sm.qbias[hq][pp][g >> 1]);
          b4[g & 1] = b4[(g & 1) + 2] = col_ok ? qs * -7.62939453125e-06f : 0.f;  // -8 * 2^-20
        }
      }
  }
  __syncthreads();

  // ------------------------------------------------------------ main loop
  // QK side: lane (g, t) holds head 4 hq + t of tokens g and g + 8 of the
  // warp's 16. PV side: columns 2t, 2t+1 are query heads 2t, 2t+1; rows are
  // dims of the warp's two cells.
  bool head_ok[HQ];
#pragma unroll
  for (int hq = 0; hq < HQ; ++hq) head_ok[hq] = G >= 4 || t < G;
  float m_run[HQ], m_ref[HQ], thr[HQ], l_run[HQ];
#pragma unroll
  for (int hq = 0; hq < HQ; ++hq) {
    m_run[hq] = -INFINITY;  // the group's running max of the scaled scores (base 2)
    m_ref[hq] = 0.f;        // exponent reference: m_run + SLACK, or 0 while m_run = -inf
    thr[hq] = -INFINITY;    // 0, or -inf while m_run = -inf: the fast path needs x - m_ref <= thr
    l_run[hq] = 0.f;
  }
  float acc[CPW][2][4];
#pragma unroll
  for (int c = 0; c < CPW; ++c)
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[c][k][i] = 0.f;
  // The -8 offset of V. head_dim 256, per-cell scales: vsum[j] = running
  // sum, over this warp's k-step of every stage, of p(token, head 2t + j) *
  // v_scale(token, cell g), the group's warps adding up at the end. Per-token
  // scales, or head_dim 128 (one cell per warp): the sum of p * v_scale over
  // every token for the warp's own cells, kept by the warp itself.
  constexpr bool OWN_SUM = VTOK || D == 128;
  float vsum[2] = {0.f, 0.f};

  // K ldmatrix (plain): matrix mi = lane / 8 covers tokens 16w + 8 (mi & 1)
  // .. +7 and cell 2 pp + (mi >> 1). The rows are 8-aligned, so the swizzle
  // of row r (128-byte rows: chunk ^= r mod 8; 64-byte rows: chunk ^=
  // (r / 2) mod 4) only depends on r mod 8 = lane mod 8.
  const int sw = lane & 7;
  const int swz = D == 256 ? sw : (sw >> 1);
  uint32_t koff[PAIRS];
#pragma unroll
  for (int pp = 0; pp < PAIRS; ++pp)
    koff[pp] = (uint32_t)((16 * gw + 8 * ((lane >> 3) & 1) + sw) * ROW_BYTES) +
               ((uint32_t)((2 * pp + (lane >> 4)) ^ swz) << 4);
  // V ldmatrix (transposed) of k-step kk: tokens 16 kk + 8 (mi & 1) .. +7,
  // cell CPW w + (mi >> 1) (head_dim 128: x2, one cell).
  const uint32_t voff = (uint32_t)((8 * ((lane >> 3) & 1) + sw) * ROW_BYTES) +
                        ((uint32_t)((CPW * gw + (D == 256 ? (lane >> 4) : 0)) ^ swz) << 4);
  const uint32_t bar_id = 1 + grp;  // the group's named barrier (0 is __syncthreads)
  bool aborted = false;
  float sg[HQ], sg8[HQ];  // raw scores of tokens g, g + 8 of the warp's 16 (head 4 hq + t)

  // Q K^T of the warp's 16 tokens of the stage in K slot `ks`.
  auto qk_math = [&](int ks) {
    const uint32_t kbase = smem_u32(&gs.k[ks][0]);
    const uint8_t* ksb = &gs.ks[ks][16 * gw * SROW_BYTES];
    uint32_t sa[PAIRS], sb[PAIRS];  // fp16 scales of cells 2pp, 2pp + 1 of tokens g, g + 8
    if constexpr (D == 256) {
      const uint4 skA = lds128(ksb + g * SROW_BYTES), skB = lds128(ksb + (g + 8) * SROW_BYTES);
      sa[0] = skA.x, sa[1] = skA.y, sa[2] = skA.z, sa[3] = skA.w;
      sb[0] = skB.x, sb[1] = skB.y, sb[2] = skB.z, sb[3] = skB.w;
    } else {
      const uint2 skA = lds64(ksb + g * SROW_BYTES), skB = lds64(ksb + (g + 8) * SROW_BYTES);
      sa[0] = skA.x, sa[1] = skA.y;
      sb[0] = skB.x, sb[1] = skB.y;
    }
#pragma unroll
    for (int pp = 0; pp < PAIRS; ++pp) {
      uint32_t kw[4];
      ldsm_x4(kbase + koff[pp], kw);  // tok g / g+8 of cell 2pp, then of cell 2pp+1
      uint32_t kh[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) kh[i] = kw[i] >> 8;
      const float2 fa = __half22float2(u32_as_h2(sa[pp])), fb = __half22float2(u32_as_h2(sb[pp]));
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) {
        const uint4 qa = sm.qfrag[hq][pp][0][lane], qb = sm.qfrag[hq][pp][1][lane];
        const float4 bias = sm.qbias[hq][pp][t];
        float d[4];
        mma_f16_c(d, kw[0] & LO4, kw[1] & LO4, kw[2] & LO4, kw[3] & LO4, qa.x, qa.y, bias.x, bias.y, bias.z,
                  bias.w);
        mma_f16(d, kw[0] & HI4, kw[1] & HI4, kw[2] & HI4, kw[3] & HI4, qa.z, qa.w);
        mma_f16(d, kh[0] & LO4, kh[1] & LO4, kh[2] & LO4, kh[3] & LO4, qb.x, qb.y);
        mma_f16(d, kh[0] & HI4, kh[1] & HI4, kh[2] & HI4, kh[3] & HI4, qb.z, qb.w);
        // columns 2t (even cell) and 2t+1 (odd cell) of head t
        sg[hq] = fmaf(fa.x, d[0], sg[hq]);
        sg[hq] = fmaf(fa.y, d[1], sg[hq]);
        sg8[hq] = fmaf(fb.x, d[2], sg8[hq]);
        sg8[hq] = fmaf(fb.y, d[3], sg8[hq]);
      }
    }
  };

  // P V of the 64 tokens of the stage in V slot `vs` (probabilities in
  // buffer `pb`) into the dims of the warp's cells (2w, 2w + 1; head_dim
  // 128: w); `partial` masks absent tokens of `smask` (a stale slot may hold
  // any bit pattern).
  auto pv_math = [&](int vs, int pb, unsigned long long smask, auto partial) {
    const uint32_t vbase = smem_u32(&gs.v[vs][0]) + voff;
    const uint8_t* vsb = &gs.vs[vs][0];
    const uint16_t* prow = &gs.prob[pb][g][0];
    auto pv_step = [&](int kk, uint32_t km) {
      const uint32_t b01 = lds32(prow + 16 * kk + 2 * t);
      const uint32_t b23 = lds32(prow + 16 * kk + 2 * t + 8);
      if constexpr (OWN_SUM) {
        // one B operand serves all of the warp's cells: one scale per token
        // (the pair of tokens 2t, 2t+1, and +8, is one word), or the one cell
        // of head_dim 128 (its half of two tokens' words)
        uint32_t s01, s89;
        if constexpr (VTOK) {
          const uint16_t* sv = reinterpret_cast<const uint16_t*>(vsb) + 16 * kk + 2 * t;
          s01 = lds32(sv), s89 = lds32(sv + 8);
        } else {
          const uint8_t* sr = vsb + (16 * kk + 2 * t) * SROW_BYTES + 4 * (gw >> 1);  // cells gw & ~1, gw | 1
          const uint32_t sel = (gw & 1) ? 0x7632u : 0x5410u;
          s01 = __byte_perm(lds32(sr), lds32(sr + SROW_BYTES), sel);
          s89 = __byte_perm(lds32(sr + 8 * SROW_BYTES), lds32(sr + 9 * SROW_BYTES), sel);
        }
        if constexpr (decltype(partial)::value) {
          s01 &= (((km >> (2 * t)) & 1u) ? 0x0000ffffu : 0u) | (((km >> (2 * t + 1)) & 1u) ? 0xffff0000u : 0u);
          s89 &= (((km >> (2 * t + 8)) & 1u) ? 0x0000ffffu : 0u) | (((km >> (2 * t + 9)) & 1u) ? 0xffff0000u : 0u);
        }
        const uint32_t b01c = h2_as_u32(__hmul2(u32_as_h2(b01), u32_as_h2(s01)));
        const uint32_t b23c = h2_as_u32(__hmul2(u32_as_h2(b23), u32_as_h2(s89)));
        uint32_t vw[4];
        if constexpr (D == 256)
          ldsm_x4_trans(vbase + (uint32_t)(16 * kk * ROW_BYTES), vw);
        else
          ldsm_x2_trans(vbase + (uint32_t)(16 * kk * ROW_BYTES), vw[0], vw[1]);
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
          const uint32_t za = vw[2 * c], zb = vw[2 * c + 1];
          const uint32_t za8 = za >> 8, zb8 = zb >> 8;
          mma_f16(acc[c][0], za & LO4, za & HI4, zb & LO4, zb & HI4, b01c, b23c);
          mma_f16(acc[c][1], za8 & LO4, za8 & HI4, zb8 & LO4, zb8 & HI4, b01c, b23c);
        }
        // the -8 offset, sum over tokens of p * v_scale per head: an MMA
        // with an all-ones A sums the B columns
        constexpr uint32_t ONES = 0x3C003C00u;  // fp16 pair (1, 1)
        float dd[4];
        mma_f16_c(dd, ONES, ONES, ONES, ONES, b01c, b23c, vsum[0], vsum[1], 0.f, 0.f);
        vsum[0] = dd[0];
        vsum[1] = dd[1];
      } else {
      const uint8_t* sr = vsb + (16 * kk + 2 * t) * SROW_BYTES + 4 * gw;  // cells 2w, 2w+1
      uint32_t s0 = lds32(sr), s1 = lds32(sr + SROW_BYTES), s2 = lds32(sr + 8 * SROW_BYTES),
               s3 = lds32(sr + 9 * SROW_BYTES);
      if constexpr (decltype(partial)::value) {
        s0 = ((km >> (2 * t)) & 1u) ? s0 : 0u;
        s1 = ((km >> (2 * t + 1)) & 1u) ? s1 : 0u;
        s2 = ((km >> (2 * t + 8)) & 1u) ? s2 : 0u;
        s3 = ((km >> (2 * t + 9)) & 1u) ? s3 : 0u;
      }
      uint32_t vw[4];
      ldsm_x4_trans(vbase + (uint32_t)(16 * kk * ROW_BYTES), vw);
#pragma unroll
      for (int c = 0; c < CPW; ++c) {
        const uint32_t sel = c ? 0x7632u : 0x5410u;
        const uint32_t b01c = h2_as_u32(__hmul2(u32_as_h2(b01), u32_as_h2(__byte_perm(s0, s1, sel))));
        const uint32_t b23c = h2_as_u32(__hmul2(u32_as_h2(b23), u32_as_h2(__byte_perm(s2, s3, sel))));
        const uint32_t za = vw[2 * c], zb = vw[2 * c + 1];
        const uint32_t za8 = za >> 8, zb8 = zb >> 8;
        mma_f16(acc[c][0], za & LO4, za & HI4, zb & LO4, zb & HI4, b01c, b23c);
        mma_f16(acc[c][1], za8 & LO4, za8 & HI4, zb8 & LO4, zb8 & HI4, b01c, b23c);
      }
      }
    };
    if constexpr (decltype(partial)::value) {
#pragma unroll
      for (int kk = 0; kk < STAGE_TOK / 16; ++kk) {
        const uint32_t km = (uint32_t)(smask >> (16 * kk)) & 0xffffu;
        if (km != 0u) pv_step(kk, km);
      }
    } else {
#pragma unroll
      for (int kk = 0; kk < STAGE_TOK / 16; ++kk) pv_step(kk, 0xffffu);
    }
    // The -8 offset: this warp sums p * v_scale over its own k-step (tokens
    // 16w .. 16w + 15) for every cell; the group's warps add up at the end.
    const uint32_t wm = (uint32_t)(smask >> (16 * gw)) & 0xffffu;
    if (!OWN_SUM && (!decltype(partial)::value || wm != 0u)) {
      const uint32_t b01 = lds32(prow + 16 * gw + 2 * t);
      const uint32_t b23 = lds32(prow + 16 * gw + 2 * t + 8);
      // A: the V scales transposed, row = cell g, k = tokens
      uint32_t st0, st1;
      ldsm_x2_trans(smem_u32(vsb) + (uint32_t)((16 * gw + (lane & 15)) * SROW_BYTES), st0, st1);
      if constexpr (decltype(partial)::value) {
        st0 &= (((wm >> (2 * t)) & 1u) ? 0x0000ffffu : 0u) | (((wm >> (2 * t + 1)) & 1u) ? 0xffff0000u : 0u);
        st1 &= (((wm >> (2 * t + 8)) & 1u) ? 0x0000ffffu : 0u) | (((wm >> (2 * t + 9)) & 1u) ? 0xffff0000u : 0u);
      }
      float dd[4];
      mma_f16_c(dd, st0, 0u, st1, 0u, b01, b23, vsum[0], vsum[1], 0.f, 0.f);
      vsum[0] = dd[0];
      vsum[1] = dd[1];
    }
  };

  // Probabilities of the scored stage (its tokens in wm) against the group's
  // running max, written to buffer pb; then the group barrier that publishes
  // them. The group's warps are then past Q K^T of that stage and P V of the
  // one before it.
  auto publish = [&](int pb, uint32_t wm) {
    const bool okA = (wm >> g) & 1u, okB = (wm >> (g + 8)) & 1u;
    float xA[HQ], xB[HQ], psum[HQ];
    bool need = false;
#pragma unroll
    for (int hq = 0; hq < HQ; ++hq) {
      xA[hq] = (okA && head_ok[hq]) ? sg[hq] * score_scale : -INFINITY;
      xB[hq] = (okB && head_ok[hq]) ? sg8[hq] * score_scale : -INFINITY;
      const float yA = xA[hq] - m_ref[hq], yB = xB[hq] - m_ref[hq];
      need |= (yA > thr[hq]) || (yB > thr[hq]);
      const float pA = ex2(yA), pB = ex2(yB);
      psum[hq] = pA + pB;
      uint16_t* pr = &gs.prob[pb][4 * hq + t][16 * gw + g];
      pr[0] = __half_as_ushort(__float2half_rn(pA));
      pr[8] = __half_as_ushort(__float2half_rn(pB));
    }
    if (bar_red_or(bar_id, need)) {
      // Some head's running max moves: exchange the tile maxima, rescale.
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) {
        float tm = fmaxf(xA[hq], xB[hq]);
        tm = fmaxf(tm, __shfl_xor_sync(FULL_MASK, tm, 4));
        tm = fmaxf(tm, __shfl_xor_sync(FULL_MASK, tm, 8));
        tm = fmaxf(tm, __shfl_xor_sync(FULL_MASK, tm, 16));
        if (g == 0) gs.tmax[gw][4 * hq + t] = tm;
      }
      bar_sync(bar_id);
      float alpha[HQ];
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) {
        float mn = m_run[hq];
#pragma unroll
        for (int w = 0; w < GWARPS; ++w) mn = fmaxf(mn, gs.tmax[w][4 * hq + t]);
        const float mu = (mn == -INFINITY) ? 0.f : mn + SLACK;
        alpha[hq] = (m_run[hq] == -INFINITY) ? 0.f : ex2(m_ref[hq] - mu);  // nothing accumulated yet: 0
        m_run[hq] = mn;
        m_ref[hq] = mu;
        thr[hq] = (mn == -INFINITY) ? -INFINITY : 0.f;
        const float pA = ex2(xA[hq] - mu), pB = ex2(xB[hq] - mu);
        l_run[hq] = l_run[hq] * alpha[hq] + (pA + pB);
        uint16_t* pr = &gs.prob[pb][4 * hq + t][16 * gw + g];
        pr[0] = __half_as_ushort(__float2half_rn(pA));
        pr[8] = __half_as_ushort(__float2half_rn(pB));
      }
      // PV columns 2t, 2t+1 are heads 2t, 2t+1: their alphas sit on the lanes
      // t' = 2t mod 4 and 2t+1 mod 4 of quad (2t) / 4.
      const int src0 = (lane & ~3) | ((2 * t) & 3), src1 = src0 | 1;
      float al0 = __shfl_sync(FULL_MASK, alpha[0], src0), al1 = __shfl_sync(FULL_MASK, alpha[0], src1);
      if (HQ > 1) {
        const float b0 = __shfl_sync(FULL_MASK, alpha[HQ - 1], src0), b1 = __shfl_sync(FULL_MASK, alpha[HQ - 1], src1);
        if (t >= 2) {
          al0 = b0;
          al1 = b1;
        }
      }
#pragma unroll
      for (int c = 0; c < CPW; ++c)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          acc[c][k][0] *= al0;
          acc[c][k][1] *= al1;
          acc[c][k][2] *= al0;
          acc[c][k][3] *= al1;
        }
      vsum[0] *= al0;
      vsum[1] *= al1;
      bar_sync(bar_id);
    } else {
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) l_run[hq] += psum[hq];
    }
  };

  // Software pipeline: iteration `it` multiplies local stage it into the
  // accumulators and scores local stage it + 1, so the two run as one
  // straight block on full stages; the group barrier sits between the
  // scoring and the P V of each stage. Local stage j + 2 is issued at the
  // barrier of local stage j. The stage count n_local is read only for stages
  // whose claim was made at least four barriers earlier, so every warp of the
  // group sees the same count.
  int kst = 0, vst = 0;       // K slot of the next local stage to score, V slot of local stage it
  uint32_t kph = 0, vph = 0;  // their phase parities
  unsigned long long smask_n = 0;  // token mask of the next stage to score
  auto next_k = [&]() {
    if (++kst == NSK) {
      kst = 0;
      kph ^= 1u;
    }
  };
  if (*n_local > 0) {
    // (aborted is warp-uniform, so the .aligned ldmatrix / mma see a converged warp)
    aborted = __any_sync(FULL_MASK, !wait_copies(&gs.kfull[0], 0, abort_flag, p.status));
    smask_n = aborted ? 0ull : gs.mask[0];
    const uint32_t wm = (uint32_t)(smask_n >> (16 * gw)) & 0xffffu;
#pragma unroll
    for (int hq = 0; hq < HQ; ++hq) sg[hq] = sg8[hq] = 0.f;
    if (wm != 0u) qk_math(0);
    publish(0, wm);
    if (gw == 2) issue(2, !aborted);
    next_k();
    for (int it = 0;; ++it) {
      const unsigned long long smask = smask_n;  // local stage it
      const bool nxt = it + 1 < *n_local;
      if (!aborted) {
        bool ok = wait_copies(&gs.vfull[vst], vph, abort_flag, p.status);
        if (nxt) ok = ok && wait_copies(&gs.kfull[kst], kph, abort_flag, p.status);
        aborted = __any_sync(FULL_MASK, !ok);
      }
      smask_n = (nxt && !aborted) ? gs.mask[kst] : 0ull;
      const uint32_t wm_n = (uint32_t)(smask_n >> (16 * gw)) & 0xffffu;
      const int pb = it & 1;
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) sg[hq] = sg8[hq] = 0.f;
      if (!aborted && smask == ~0ull && (smask_n == ~0ull || !nxt)) {
        // full stages: one straight block
        pv_math(vst, pb, smask, std::false_type{});
        if (nxt) qk_math(kst);
      } else {
        if (!aborted && smask != 0ull) pv_math(vst, pb, smask, std::true_type{});
        if (wm_n != 0u) qk_math(kst);
      }
      if (!nxt) break;
      publish(pb ^ 1, wm_n);
      // local stage it + 3 takes the K slot of stage it + 1 (scored) and the
      // V slot of stage it (multiplied); its claim is kept going even when
      // aborting, so that the stage count gets set.
      if (((it + 3) % GWARPS) == gw) issue(it + 3, !aborted);
      next_k();
      if (++vst == NSV) {
        vst = 0;
        vph ^= 1u;
      }
    }
  }

  // ------------------------------------------------------------ epilogue
  // Per group: softmax sums of the warps, offset sums of the warps (in the
  // group's idle V scale slots), and the decoded accumulators.
#pragma unroll
  for (int hq = 0; hq < HQ; ++hq) {
    float l = l_run[hq];
    l += __shfl_xor_sync(FULL_MASK, l, 4);
    l += __shfl_xor_sync(FULL_MASK, l, 8);
    l += __shfl_xor_sync(FULL_MASK, l, 16);
    if (g == 0) gs.wl[gw][4 * hq + t] = l;
  }
  __syncthreads();
  if (*abort_flag) {
    // Leave only after every copy issued here has landed.
    if (threadIdx.x < GROUPS) {
      GroupSmem<D>& q = sm.grp[threadIdx.x];
      const int issued = q.issued;
      for (int r = max(0, issued - NSK); r < issued; ++r)
        if (!mbar_wait_bounded(&q.kfull[r % NSK], (r / NSK) & 1)) flag(p.status, QKV_DEV_TIMEOUT);
      for (int r = max(0, issued - NSV); r < issued; ++r)
        if (!mbar_wait_bounded(&q.vfull[r % NSV], (r / NSV) & 1)) flag(p.status, QKV_DEV_TIMEOUT);
    }
    if (threadIdx.x < G) lse_out[threadIdx.x] = -INFINITY;
  } else {
    float2* vsp = reinterpret_cast<float2*>(&gs.vs[0][0]);  // (head_dim 256, per-cell scales)
    if constexpr (!OWN_SUM) vsp[gw * 32 + lane] = make_float2(vsum[0], vsum[1]);
    bar_sync(bar_id);
    // the group's softmax sum and exponent reference per head
    if (gw == 0 && g == 0) {
#pragma unroll
      for (int hq = 0; hq < HQ; ++hq) {
        const int h = 4 * hq + t;
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < GWARPS; ++w) Ls += gs.wl[w][h];
        sm.gl[grp][h] = Ls;
        sm.gm[grp][h] = m_ref[hq];
      }
    }
    // Undo the subnormal encoding of V: rows 0-7 carry 2^-24 * sum(n p s),
    // rows 8-15 2^-20 * sum(n p s); the -8 offset is 8 * sum(p s) per cell.
#pragma unroll
    for (int c = 0; c < CPW; ++c) {
      const int cell = CPW * gw + c;
      float b0 = 0.f, b1 = 0.f;
      if constexpr (OWN_SUM) {  // the warp's own sum covers every token of its cells
        b0 = vsum[0];
        b1 = vsum[1];
      } else {
#pragma unroll
        for (int w = 0; w < GWARPS; ++w) {
          const float2 v = vsp[w * 32 + 4 * cell + t];
          b0 += v.x;
          b1 += v.y;
        }
      }
      b0 *= 8.f;
      b1 *= 8.f;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        acc[c][k][0] = fmaf(acc[c][k][0], 16777216.f, -b0);
        acc[c][k][1] = fmaf(acc[c][k][1], 16777216.f, -b1);
        acc[c][k][2] = fmaf(acc[c][k][2], 1048576.f, -b0);
        acc[c][k][3] = fmaf(acc[c][k][3], 1048576.f, -b1);
      }
    }
    __syncthreads();
    // Fold the groups: weights 2^(m_ref of the group - M) per head.
    // [group][head][D + 4 dims], in group 0's idle rings: the 4-float pad
    // puts the heads of one quarter-warp's stores in different banks
    constexpr int SLAB_ROW = D + 4;
    static_assert(GROUPS * 8 * SLAB_ROW * 4 <= (NSK + NSV) * STAGE_TOK * Geo<D>::ROW_BYTES, "slab fits the rings");
    float* slab = reinterpret_cast<float*>(&sm.grp[0].k[0][0]);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int h = 2 * t + j;
      if (h < G) {
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < GROUPS; ++q)
          if (sm.gl[q][h] > 0.f) M = fmaxf(M, sm.gm[q][h]);
        const float f = (sm.gl[grp][h] > 0.f) ? exp2f(sm.gm[grp][h] - M) : 0.f;
        float* dst = slab + ((size_t)grp * G + h) * SLAB_ROW + 4 * g;
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
          const float4 o = make_float4(f * acc[c][0][j], f * acc[c][0][j + 2], f * acc[c][1][j], f * acc[c][1][j + 2]);
          *reinterpret_cast<float4*>(dst + 32 * (CPW * gw + c)) = o;
        }
      }
    }
    __syncthreads();
    // Sum the groups, normalise, write the partial of this split.
    for (int e = threadIdx.x; e < G * (D / 4); e += THREADS) {
      const int h = e / (D / 4), d4 = e % (D / 4);
      float M = -INFINITY;
#pragma unroll
      for (int q = 0; q < GROUPS; ++q)
        if (sm.gl[q][h] > 0.f) M = fmaxf(M, sm.gm[q][h]);
      float Ls = 0.f;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < GROUPS; ++q) {
        const float f = (sm.gl[q][h] > 0.f) ? exp2f(sm.gm[q][h] - M) : 0.f;
        Ls = fmaf(f, sm.gl[q][h], Ls);
        const float4 x = *reinterpret_cast<const float4*>(slab + ((size_t)q * G + h) * SLAB_ROW + 4 * d4);
        o.x += x.x;
        o.y += x.y;
        o.z += x.z;
        o.w += x.w;
      }
      const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
      o.x *= inv;
      o.y *= inv;
      o.z *= inv;
      o.w *= inv;
      *reinterpret_cast<float4*>(p.o_parts + ((size_t)split * rows + row0 + h) * D + 4 * d4) = o;
      if (d4 == 0) lse_out[h] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
    }
  }
}


// The kernel instance for (block, G, per-token V scales, decode step) at
// head_dim D, or nullptr for a shape not compiled, and its dynamic shared
// memory. decode_split.cu instantiates D = 256, decode_split_d128.cu D = 128
// (one translation unit each, so that they compile in parallel).
template <int D, int BLOCK, int G>
const void* split_kernel_of(bool vtok, bool fuse) {
  if (fuse)
    return vtok ? reinterpret_cast<const void*>(&paged_decode_split_kernel<D, BLOCK, G, true, true>)
                : reinterpret_cast<const void*>(&paged_decode_split_kernel<D, BLOCK, G, false, true>);
  return vtok ? reinterpret_cast<const void*>(&paged_decode_split_kernel<D, BLOCK, G, true, false>)
              : reinterpret_cast<const void*>(&paged_decode_split_kernel<D, BLOCK, G, false, false>);
}

template <int D>
const void* split_kernel(int block, int G, bool vtok, bool fuse) {
#define QKV_PICK(B)                                                    \
  if (block == B) {                                                    \
    if (G == 1) return split_kernel_of<D, B, 1>(vtok, fuse);           \
    if (G == 2) return split_kernel_of<D, B, 2>(vtok, fuse);           \
    if (G == 4) return split_kernel_of<D, B, 4>(vtok, fuse);           \
    if (G == 8) return split_kernel_of<D, B, 8>(vtok, fuse);           \
  }
  QKV_PICK(16)
  QKV_PICK(32)
  QKV_PICK(64)
#undef QKV_PICK
  return nullptr;
}

template <int D>
size_t split_kernel_smem(int G) {
  return G > 4 ? smem_bytes<2, D>() : smem_bytes<1, D>();
}

}  // namespace qkv
