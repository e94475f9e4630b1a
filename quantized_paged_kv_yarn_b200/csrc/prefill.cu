// prefill.cu -- chunked causal prefill attention over the paged F4 cache
// on the sm_100a tensor cores (tcgen05, CTA pairs, accumulators in tensor
// memory).
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2
// (the packed cache, values (nibble - 8) * scale) and section 5 (paged
// prefill in chunks of 2048 tokens). A chunk of n_q queries of one sequence
// sits at cache tokens prefix_len .. prefix_len + n_q - 1 (already written);
// query i attends the cached tokens 0 .. prefix_len + i.
//
// This is a dense contraction (256 query rows share every dequantised
// page), so it runs on tcgen05.mma with fp32 accumulators in TMEM, issued
// for a pair of CTAs on two SMs (cta_group::2, M = 256). With head_dim D
// (256 or 128):
//
//   S[256 x 64] = Q'[256 x D] . (K^'hi + K^'lo)[64 x D]^T   (D/16 MMAs, K = 16, N = 128)
//   O[256 x D] += P[256 x 64] . V^'[64 x D]                 (4 MMAs, N = D)
//
// The hi and lo tiles of K^' stand side by side as one B operand of 128
// rows, so Q K^T takes D/16 MMAs of N = 128 instead of 2 D/16 of N = 64 (on
// this part an N = 64 MMA takes 45 cycles, an N = 128 one 64); the softmax
// adds the two products of each token.
//
// Rows are (query head of the GQA group, query): 256 = G x (256 / G); CTA
// rank r of the pair owns rows 128 r .. 128 r + 127 (its rows of the Q'
// tile, its lanes of S, P and O). The B operands are split by N: of each
// 64-token stage, rank r dequantises the K of tokens 32 r .. 32 r + 31 (all
// D dims) and the V of dims D/2 r .. D/2 r + D/2 - 1 (all 64 tokens) into
// its own shared memory,
// so each SM writes and the tensor core reads half of every tile, and the
// shared-memory pipe (the bound of a one-SM version) carries half the bytes.
// One pair per (256 / G queries, KV head).
//
// Warp roles (512 threads per CTA):
//   warp 0        TMEM allocation (both CTAs); in rank 0, lane 0 issues every
//                 MMA and commit of the pair
//   warps 4..7    softmax: thread r owns row r of its CTA (TMEM lane r): puts
//                 its row of Q' into shared memory, reads S, keeps the running
//                 max and sum, writes P, rescales O when the max moves, and
//                 writes the output
//   warps 8..11   K dequantisation: D/4 dims of one token's K per thread
//   warps 12..15  V dequantisation: D/4 of one token's D/2 dims of this CTA
//                 Packed bytes are read two stages ahead, page ids one
//                 load ahead of those.
// Producers signal rank 0's barriers (a remote arrive from rank 1); the MMA
// thread's commits arrive on both CTAs' barriers (multicast).
//
// Numerics. With s' = scale * 2^-4 (exact while scale >= 2^-10; the 2^-4
// keeps 8 * 65504 in range), a K element (code - 8) s' needs up to 14
// significant bits: it is split into K^'hi = fp16((code - 8) s') and
// K^'lo = fp16((code - 8) s' - K^'hi), and their sum is exact, so the
// scores see K exactly (one fp16 rounding of K alone moved scores by up to
// ~1e-3, more than the attention tolerance allows at short contexts).
// V^' = fp16((code - 8) s') is rounded once. Q' = fp16(q * 2^e) with a power
// of two per row (exact for bf16 q in range). The hi and lo products of a
// score accumulate apart in fp32 and are added in fp32, P . V accumulates
// in fp32; p = 2^(s - m_ref) in fp16 with the reference max moved
// lazily (only when a score exceeds it by more than 8, so p <= 256).
//
// P lives in tensor memory (the A operand of P . V; row r in lane r, two
// fp16 per column) and overwrites the first quarter of the S columns it was
// computed from, which the next Q K^T into that slot may overwrite only
// after the P . V reading it (issued earlier by the same thread, and the
// tensor core keeps one thread's MMAs in order). Shared-memory tiles use the
// 128-byte swizzle in the canonical UMMA layouts: the K^' tiles (K-major)
// are [D/64 chunks of 64 dims][32 tokens' hi, then their lo][128 B]; Q'
// (K-major, the A operand of Q K^T) is [D/64 chunks][128 rows][128 B]; the
// V^' tile, the MN-major B operand of P . V, is [D/128 chunks of 64
// dims][64 tokens][128 B]. Within each 8-dim unit the dims are stored in
// the order 0,4,1,5,2,6,3,7 (the order in which four nibble masks of a
// packed word yield them); Q' uses the same order, and the output
// un-permutes O's columns.
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace qkv {
namespace prefill {

constexpr int THREADS = 512;
constexpr int M = 256;          // rows per CTA pair
constexpr int ML = 128;         // rows per CTA
constexpr int NT = 64;          // tokens per stage
constexpr int NTL = NT / 2;     // K tokens per CTA per stage
constexpr int NS = 3;           // shared-memory slots of K^ and V^
constexpr float TH = 8.f;       // lazy-rescale threshold (log2 units)

// Sizes that follow from the head dim D.
template <int D>
struct Geo {
  static_assert(D == 256 || D == 128, "head_dim 256 or 128");
  // shared-memory map (offsets from a 1024-byte aligned base)
  static constexpr int KT = (D / 64) * NTL * 128;   // the hi (or lo) rows of a K^ slot: D/64 x [32][128 B]
  static constexpr int VT = (D / 128) * NT * 128;   // one V^ tile: [D/128][64][128 B]
  static constexpr int K_OFF = 0;                   // NS slots of [D/64][hi 32 rows, lo 32 rows][128 B]
  static constexpr int V_OFF = K_OFF + NS * 2 * KT;  // NS slots
  static constexpr int Q_OFF = V_OFF + NS * VT;      // Q' of this CTA's rows: [D/64][128 rows][128 B]
  static constexpr int BAR_OFF = Q_OFF + (D / 64) * ML * 128;
  // barriers, flags and alignment slack; at least 117 KB, so that no two
  // CTAs share an SM (the tensor memory is allocated whole)
  static constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024 > 117 * 1024 ? BAR_OFF + 256 + 1024 : 117 * 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory of one CTA");
  // TMEM columns (each CTA, its 128 rows): O 0..D-1, S slot b at D + 128 b
  // (columns 0..31 the hi products of rank 0's tokens, 32..63 their lo
  // products, 64..127 the same for rank 1's; P of that stage, fp16,
  // overwrites the first 32 columns once S is read)
  static constexpr uint32_t TS = D;
  // dims one dequantising thread converts per stage, and its 16-byte units
  static constexpr int DPT = D / 4;
  static constexpr int UPT = DPT / 8;
};
constexpr uint32_t TMEM_COLS = 512;
static_assert(Geo<256>::TS + 4 * NT <= TMEM_COLS && Geo<128>::TS + 4 * NT <= TMEM_COLS, "tensor memory map");

struct Bars {
  // signalled by producers of both CTAs, waited on in rank 0. P of stage i
  // signals pready[i % 2]: with one barrier, the softmax of one CTA (which
  // needs only its own S) could finish stage i + 1 before its partner
  // finished stage i, and its arrivals would complete stage i's phase.
  // (tests/test_prefill_protocol.py models these roles and barriers and
  // checks every wait's phase over skewed schedules.)
  uint64_t kready[NS], vready[NS], pready[2], qready;
  // signalled by the MMA commits of the pair, waited on in each CTA
  uint64_t kfree[NS], vfree[NS], sfull[2], odone, drain;
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

struct Params {
  const uint16_t* q;
  uint16_t* out;
  float* lse2;
  const uint8_t* k_data;
  const uint16_t* k_scale;
  const uint8_t* v_data;
  const uint16_t* v_scale;
  const int32_t* page_table;
  int64_t num_pages;
  int n_q, prefix_len, q_heads, kv_heads, G, QB, block, block_shift, v_tok;
  int kv_limit;  // tokens past this one are not attended (a window pass: every query sees all of them)
  float score_scale;  // softmax_scale * log2(e)
  int32_t* status;
  // Context split in n_splits parts (blockIdx.z): with n_splits > 1 each
  // part writes its normalised partial output (fp32) and lse2 to o_part /
  // lse_part [part][n_q * q_heads], which the log2-sum-exp merge folds.
  int n_splits;
  float* o_part;
  float* lse_part;
};

__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  // start >> 4 | LBO >> 4 << 16 | SBO >> 4 << 32 | version 1 << 46 | 128-byte swizzle (2) << 61
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// Pair MMA: A from tensor memory (row r of each CTA in its lane r), B from
// both CTAs' shared memory at the same offset (each holds N / 2 columns).
__device__ __forceinline__ void umma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

// Pair MMA with A and B from shared memory (A: each CTA its M / 2 rows; B:
// each CTA N / 2 columns, at the same offsets in both CTAs).
__device__ __forceinline__ void umma2_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// Arrive, once the pair's MMAs issued so far are done, on the barrier at
// this offset in both CTAs.
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((unsigned short)3)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on rank 0's copy of a barrier (release at cluster scope).
__device__ __forceinline__ void arrive_rank0(uint64_t* bar) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(remote) : "r"(smem_u32(bar)));
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

#define QKV_R32(p) \
  "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3]), "=r"(p[4]), "=r"(p[5]), "=r"(p[6]), "=r"(p[7]), "=r"(p[8]), \
  "=r"(p[9]), "=r"(p[10]), "=r"(p[11]), "=r"(p[12]), "=r"(p[13]), "=r"(p[14]), "=r"(p[15]), "=r"(p[16]),       \
  "=r"(p[17]), "=r"(p[18]), "=r"(p[19]), "=r"(p[20]), "=r"(p[21]), "=r"(p[22]), "=r"(p[23]), "=r"(p[24]),      \
  "=r"(p[25]), "=r"(p[26]), "=r"(p[27]), "=r"(p[28]), "=r"(p[29]), "=r"(p[30]), "=r"(p[31])
#define QKV_W32(p) \
  "r"(p[0]), "r"(p[1]), "r"(p[2]), "r"(p[3]), "r"(p[4]), "r"(p[5]), "r"(p[6]), "r"(p[7]), "r"(p[8]), "r"(p[9]), \
  "r"(p[10]), "r"(p[11]), "r"(p[12]), "r"(p[13]), "r"(p[14]), "r"(p[15]), "r"(p[16]), "r"(p[17]), "r"(p[18]),  \
  "r"(p[19]), "r"(p[20]), "r"(p[21]), "r"(p[22]), "r"(p[23]), "r"(p[24]), "r"(p[25]), "r"(p[26]), "r"(p[27]),  \
  "r"(p[28]), "r"(p[29]), "r"(p[30]), "r"(p[31])
#define QKV_REGLIST32                                                                                           \
  "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, " \
  "%23, %24, %25, %26, %27, %28, %29, %30, %31}"

// 32 consecutive fp32 columns of this thread's TMEM lane (warp quarter rule:
// the address carries lane base 32 * (warp % 4) in its upper half)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 " QKV_REGLIST32 ", [%32];" : QKV_R32(r) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
               "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
               ::"r"(taddr), QKV_W32(r)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 2^x (hardware approximation; subnormal results flushed to 0, 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte unit u of row r in a [rows][128 B] 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t swz(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// try_wait (acquire at cluster scope: producers of the other CTA release to
// it) that may suspend the thread, using no issue slots, for up to `ns`
// nanoseconds or until the phase completes.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Give up the pair's work: this CTA's abort flag and the peer CTA's (a
// store to its shared memory through the cluster window), so that the
// roles of both CTAs stop waiting at once instead of at their own limits.
__device__ __forceinline__ void abort_pair(int* abort) {
  *reinterpret_cast<volatile int*>(abort) = 1;
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(abort)), "r"(cluster_rank() ^ 1u));
  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(1u) : "memory");
}

// Bounded wait that also gives up once another role of this CTA, or of the
// peer CTA, has aborted. Waiting threads sleep in the barrier instead of
// spinning.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > WAIT_LIMIT_NS) return false;
  }
}

// Four fp16 pairs of one packed word (8 codes, low nibble first) times the
// cell scale s' (fp16 pair): pairs (e0,e4), (e1,e5), (e2,e6), (e3,e7).
// With LO, also the rounding residual (code - 8) s' - hi (exact, one fma).
template <bool LO>
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 s2, uint32_t (&o)[4], uint32_t (&lo)[4]) {
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));  // 1032
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = ((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u;  // fp16 1024 + code, twice
    const __half2 t = __hsub2(u32_as_h2(x), off);                       // code - 8, exact
    const __half2 hi = __hmul2(t, s2);
    o[i] = h2_as_u32(hi);
    if constexpr (LO) lo[i] = h2_as_u32(__hfma2(t, s2, __hneg2(hi)));
  }
}

__device__ __forceinline__ uint32_t bf2_u32(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Loads issued where they stand in the program (volatile: the compiler may
// not sink them to their first use, which would expose their latency).
__device__ __forceinline__ uint4 ldg_early16(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint32_t ldg_early4(const void* ptr) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ uint32_t ldg_early2(const void* ptr) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(ptr));
  return v;
}

// One dequantising thread's packed bytes of one stage.
struct Raw {
  uint4 a, b;     // 32 packed bytes: 64 dims
  uint32_t sc;    // fp16 scales of the two 32-dim cells (or the token's V scale, twice)
  int ok;         // 0: outside the context (zero rows), 1: data, 2: bad page (zero rows, flagged)
  int32_t page;   // page id of the stage this set loads next (read one load ahead)
};

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    paged_prefill_kernel(const Params p) {
  using Gm = Geo<D>;
  constexpr int KT = Gm::KT, VT = Gm::VT, K_OFF = Gm::K_OFF, V_OFF = Gm::V_OFF, Q_OFF = Gm::Q_OFF;
  constexpr int BAR_OFF = Gm::BAR_OFF;
  constexpr uint32_t TS = Gm::TS;
  // 1024-aligned by pointer arithmetic on the shared array (keeps accesses in
  // the shared window)
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Bars& bars = *reinterpret_cast<Bars*>(sm + BAR_OFF);
  const uint32_t s_base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = (int)cluster_rank();

  const int kvh = blockIdx.y;
  const int QB2 = p.QB;  // queries per pair
  const int q0 = (blockIdx.x >> 1) * QB2;
  const int q_last = min(p.n_q, q0 + QB2) - 1;
  const int kv_len = min(p.prefix_len + q_last + 1, p.kv_limit);
  // this part's stages st0 .. st0 + n_st - 1 of the pair's context (the
  // host keeps n_splits <= the stage count, so every part has a stage)
  const int n_all = (kv_len + NT - 1) / NT;
  const int st0 = (int)((int64_t)blockIdx.z * n_all / p.n_splits);
  const int n_st = (int)((int64_t)(blockIdx.z + 1) * n_all / p.n_splits) - st0;

  if (tid == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(&bars.kready[b], 2 * 128);
      mbar_init(&bars.vready[b], 2 * 128);
      mbar_init(&bars.kfree[b], 1);
      mbar_init(&bars.vfree[b], 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(&bars.sfull[b], 1);
    for (int b = 0; b < 2; ++b) mbar_init(&bars.pready[b], 2 * 128);
    mbar_init(&bars.qready, 2 * 128);
    mbar_init(&bars.odone, 1);
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  // Tensor memory is taken only after the wait: the CTA holds none of the
  // SM's tensor memory (nor its allocation permit) while the kernel ahead of
  // it in the stream still runs.
  pdl_wait();
  pdl_release();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars.tmem)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = bars.tmem;
  volatile int* abort = &bars.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issue (rank 0)
    if (rank == 0 && lane == 0) {
      // Q K^T with N = 2 NT: K^'hi and K^'lo side by side as one B operand
      constexpr uint32_t ID_QK = (1u << 4) | ((uint32_t)((2 * NT) >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
      constexpr uint32_t ID_PV = (1u << 4) | (1u << 16) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
      bool ok = wait_bar(&bars.qready, 0, abort);
      // descriptors of slot 0 at offset 0; each MMA adds its byte offset >> 4
      // to the start-address field (no carry: smem offsets stay below 2^18)
      const uint64_t dv0 = sdesc(s_base + V_OFF, NT * 128, 1024);
      const uint64_t dk0 = sdesc(s_base + K_OFF, 16, 1024);
      const uint64_t dq0 = sdesc(s_base + Q_OFF, 16, 1024);
      auto pv = [&](int i) -> bool {
        const int b = i % NS, u = i / NS, sb = i & 1;
        if (!wait_bar(&bars.pready[i & 1], (uint32_t)(i >> 1) & 1u, abort)) return false;
        if (!wait_bar(&bars.vready[b], (uint32_t)u & 1u, abort)) return false;
        tc_fence_after();
        const uint64_t dv = dv0 + (uint64_t)((b * VT) >> 4);
#pragma unroll
        for (int kk = 0; kk < NT / 16; ++kk)  // A = P in tensor memory (S slot sb)
          umma2_ts(tmem, tmem + TS + 2 * NT * sb + 8 * kk, dv + (uint64_t)((2048 * kk) >> 4), ID_PV,
                   (i > 0 || kk > 0) ? 1u : 0u);
        umma2_commit_both(&bars.odone);
        umma2_commit_both(&bars.vfree[b]);
        return true;
      };
      for (int j = 0; ok && j < n_st; ++j) {
        const int b = j % NS, u = j / NS, sb = j & 1;
        if (!wait_bar(&bars.kready[b], (uint32_t)u & 1u, abort)) { ok = false; break; }
        // S slot sb is free again: P . V of stage j - 2, which read P from it,
        // was issued (after its pready) before this Q K^T, and the tensor
        // core runs one thread's MMAs in order
        tc_fence_after();
        const uint64_t dk = dk0 + (uint64_t)((b * 2 * KT) >> 4);
        const uint32_t ts = tmem + TS + 2 * NT * sb;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // 16 dims per MMA: 32 bytes into a 128-byte row
          const uint32_t koff = (kk >> 2) * (2 * NTL * 128) + 32 * (kk & 3);
          const uint32_t qoff = (kk >> 2) * (ML * 128) + 32 * (kk & 3);
          umma2_ss(ts, dq0 + (uint64_t)(qoff >> 4), dk + (uint64_t)(koff >> 4), ID_QK, kk > 0 ? 1u : 0u);
        }
        umma2_commit_both(&bars.sfull[sb]);
        umma2_commit_both(&bars.kfree[b]);
        if (j >= 1 && !pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = pv(n_st - 1);
      if (!ok) {
        abort_pair(&bars.abort);
        flag(p.status, QKV_DEV_TIMEOUT);
      }
      // every MMA issued so far has completed once this commit lands (both CTAs)
      umma2_commit_both(&bars.drain);
    }
    // both CTAs: the pair's MMAs, which write this CTA's tensor memory, are done
    if (lane == 0) mbar_wait_bounded(&bars.drain, 0);
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ softmax
    const int r = tid - 128;
    const int R = ML * rank + r;  // row of the pair
    const int hl = R / QB2, qq = R - hl * QB2;
    const int qi = q0 + qq;
    const bool valid = qi < p.n_q;
    const int qhead = kvh * p.G + hl;
    const int lim = min(p.prefix_len + qi, p.kv_limit - 1);  // last token this row attends
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

    // Q' = fp16(q * 2^e) into row r of this CTA's Q' tile, dims permuted per 8-dim unit
    float c_row;
    {
      const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)qi * p.q_heads + qhead) * D);
      float amax = 0.f;
      if (valid) {
#pragma unroll 4
        for (int u = 0; u < D / 8; ++u) {
          const uint4 w = src[u];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(ws[i] << 16)), fabsf(__uint_as_float(ws[i] & 0xffff0000u))));
        }
      }
      // 2^e with amax * 2^e in [2^13, 2^14); exponent of amax from its bits
      int e = 0;
      if (amax > 0.f) e = 13 - (((int)(__float_as_uint(amax) >> 23) & 0xff) - 127);
      e = max(-100, min(100, e));
      // 2^e as a product of two normal powers of two (|e| <= 100)
      const float up = __int_as_float((127 + e / 2) << 23) * __int_as_float((127 + (e - e / 2)) << 23);
      c_row = p.score_scale * 16.f / up;  // S = S' * 2^(4 - e)
#pragma unroll 1
      for (int g = 0; g < D / 64; ++g) {  // one 128-byte row of a 64-dim chunk
#pragma unroll
        for (int uu = 0; uu < 8; ++uu) {
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (valid) w = src[8 * g + uu];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          float f[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(ws[i] << 16) * up;
            f[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u) * up;
          }
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = h2_as_u32(__floats2half2_rn(f[i], f[i + 4]));
          sts128(s_base + Q_OFF + g * (ML * 128) + swz(r, uu), o[0], o[1], o[2], o[3]);
        }
      }
      fence_async_smem();  // the tensor core reads the tile through the async proxy
      arrive_rank0(&bars.qready);
    }

    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_st; ++j) {
      const int sb = j & 1;
      ok = wait_bar(&bars.sfull[sb], (uint32_t)(j >> 1) & 1u, abort);
      if (!__all_sync(FULL_MASK, ok)) { ok = false; break; }
      tc_fence_after();
      // score of token i = hi + lo products: columns 64 h + i % 32 and 64 h + 32 + i % 32 (h = i / 32)
      const uint32_t ts = tmem + lane_base + TS + 2 * NT * sb;
      float s[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sr[2][32];
        tmem_ld32(ts + 64 * h, sr[0]);
        tmem_ld32(ts + 64 * h + 32, sr[1]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[32 * h + i] = __uint_as_float(sr[0][i]) + __uint_as_float(sr[1][i]);
      }
      const int base = (st0 + j) * NT;
      if (base + NT - 1 > lim) {
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = (base + i <= lim) ? s[i] : -INFINITY;
      }
      float smax = s[0];
#pragma unroll
      for (int i = 1; i < 64; ++i) smax = fmaxf(smax, s[i]);
      const float mt = smax * c_row;
      const bool need = mt > m_ref + TH;
      const bool any_need = __any_sync(FULL_MASK, need);
      float alpha = 1.f;
      if (any_need) {
        const float m_new = need ? mt : m_ref;
        alpha = need ? ex2(m_ref - m_new) : 1.f;  // nothing accumulated yet: ex2(-inf) = 0
        l *= alpha;
        m_ref = m_new;
      }
      // p = 2^(s c - m_ref) as fp16 pairs (token order), summed as rounded
      const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pw[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float a = ex2(fmaf(s[2 * i], c_row, -mu));
        const float bq = ex2(fmaf(s[2 * i + 1], c_row, -mu));
        const __half2 h = __floats2half2_rn(a, bq);
        const float2 hf = __half22float2(h);
        l += hf.x + hf.y;
        pw[i] = h2_as_u32(h);
      }
      // P into the first 32 columns of S slot sb (its S is in registers)
      tmem_st32(ts, pw);
      if (any_need && j >= 1) {  // rescale O once P . V of the previous stage is done
        ok = wait_bar(&bars.odone, (uint32_t)(j - 1) & 1u, abort);
        if (!__all_sync(FULL_MASK, ok)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + 32 * c, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      arrive_rank0(&bars.pready[j & 1]);
    }

    // epilogue: O / l, columns un-permuted; bf16 out, or this part's fp32 partial.
    // O is complete once the drain commit lands (one phase, after every MMA of
    // the pair). A parity wait on odone cannot say so: P . V of stage n_st - 2
    // is issued after the last Q K^T, so odone may still be in phase n_st - 2,
    // whose parity differs from that of n_st - 1, and the wait would return
    // before the last two P . V products are in O.
    if (ok) {
      ok = wait_bar(&bars.drain, 0u, abort) && !*abort;
      ok = __all_sync(FULL_MASK, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 16.f / l : 0.f;
      const size_t row = (size_t)qi * p.q_heads + qhead;
      const bool part = p.o_part != nullptr;
      uint16_t* dst = p.out + row * D;
      float* pdst = part ? p.o_part + ((size_t)blockIdx.z * p.n_q * p.q_heads + row) * D : nullptr;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + 32 * c, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {  // columns 8u .. 8u+7 hold dims 8u + (0,4,1,5,2,6,3,7)
            float f[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              f[k] = __uint_as_float(o[8 * u + 2 * k]) * inv;
              f[k + 4] = __uint_as_float(o[8 * u + 2 * k + 1]) * inv;
            }
            if (part) {
              reinterpret_cast<float4*>(pdst)[2 * (4 * c + u)] = make_float4(f[0], f[1], f[2], f[3]);
              reinterpret_cast<float4*>(pdst)[2 * (4 * c + u) + 1] = make_float4(f[4], f[5], f[6], f[7]);
            } else {
              reinterpret_cast<uint4*>(dst)[4 * c + u] =
                  make_uint4(bf2_u32(f[0], f[1]), bf2_u32(f[2], f[3]), bf2_u32(f[4], f[5]), bf2_u32(f[6], f[7]));
            }
          }
        }
      }
      const float lse = l > 0.f ? m_ref + log2f(l) : -INFINITY;
      if (valid && part) p.lse_part[(size_t)blockIdx.z * p.n_q * p.q_heads + row] = lse;
      else if (valid && p.lse2) p.lse2[row] = lse;
    } else {
      abort_pair(&bars.abort);
      flag(p.status, QKV_DEV_TIMEOUT);
    }
    tc_fence_before();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dequantisation
    constexpr int DPT = Gm::DPT, UPT = Gm::UPT;
    const bool is_k = warp < 12;
    const int d = is_k ? tid - 256 : tid - 384;  // 0..127
    // K: row d % 8 + 8 (d / 32) of this CTA's 32 tokens, dims DPT ((d / 8) % 4) .. + DPT - 1
    // V: token d % 8 + 8 (d / 16) of the stage, dims D/2 rank + DPT ((d / 8) % 2) .. + DPT - 1
    // The eight lanes of a quarter-warp take eight consecutive rows: their
    // 16-byte stores (a quarter-warp per shared-memory wavefront) land in
    // eight different 16-byte columns of the swizzled tile, one wavefront
    // each (with the dim slot as the fastest index, four lanes of a quarter
    // hit the same column: 16 wavefronts per K store, 8 per V store).
    const int trow = is_k ? (d & 7) + 8 * (d >> 5) : (d & 7) + 8 * (d >> 4);  // row in this CTA's tile
    const int tk = is_k ? NTL * rank + trow : trow;
    const int slot = is_k ? ((d >> 3) & 3) : ((d >> 3) & 1);
    const int tdim = DPT * slot;       // first dim in the tile (K: of D, V: of this CTA's D/2)
    const int chunk = tdim / 64;       // 64-dim chunk of the tile
    const int unit0 = (tdim % 64) / 8;  // first 16-byte unit in the chunk's row
    const int byte_off = (is_k ? tdim : (D / 2) * rank + tdim) / 2;  // in the packed row
    const int cell = byte_off / 16;                                   // first 32-dim cell
    const uint8_t* data = is_k ? p.k_data : p.v_data;
    const uint16_t* scales = is_k ? p.k_scale : p.v_scale;
    const bool per_tok = !is_k && p.v_tok;
    const size_t row_bytes = D / 2;
    // page id of this thread's token in stage j (-1 past the context)
    auto page_of = [&](int j) -> int32_t {
      const int t = (st0 + j) * NT + tk;
      return (j < n_st && t < kv_len) ? (int32_t)ldg_early4(p.page_table + (t >> p.block_shift)) : -1;
    };
    // The packed bytes of stage j into x, using the page id read by the
    // previous load of x; then the page id of stage j + 2 for the next one,
    // so no data load waits on a page-table read.
    auto load = [&](int j, Raw& x) {
      const int32_t page = x.page;
      x.page = page_of(j + 2);
      x.ok = 0;
      const int t = (st0 + j) * NT + tk;
      if (j >= n_st || t >= kv_len) return;
      if (page < 0 || page >= p.num_pages) {
        x.ok = 2;
        return;
      }
      const size_t row = ((size_t)page * p.kv_heads + kvh) * p.block + (t & (p.block - 1));
      const uint4* src = reinterpret_cast<const uint4*>(data + row * row_bytes + byte_off);
      x.a = ldg_early16(src);
      if constexpr (UPT == 8) x.b = ldg_early16(src + 1);
      if (per_tok) {
        const uint32_t h = ldg_early2(scales + row);
        x.sc = h | (h << 16);
      } else if constexpr (UPT == 8) {
        x.sc = ldg_early4(scales + row * (D / 32) + cell);  // two cells (cell is even)
      } else {
        const uint32_t h = ldg_early2(scales + row * (D / 32) + cell);
        x.sc = h | (h << 16);
      }
      x.ok = 1;
    };
    // this thread's DPT dims of one token into its units of a tile slot (K: hi and lo tiles)
    auto put = [&](uint32_t chunk_base, const Raw& x, auto with_lo) {
      constexpr bool LO = decltype(with_lo)::value;
      // s' = scale * 2^-4 per cell (low half: first cell, high half: second)
      const __half2 s16 = __hmul2(u32_as_h2(x.sc), __halves2half2(__ushort_as_half(0x2C00), __ushort_as_half(0x2C00)));
      const __half2 s_lo = __low2half2(s16), s_hi = __high2half2(s16);
      const uint32_t wd[8] = {x.a.x, x.a.y, x.a.z, x.a.w, x.b.x, x.b.y, x.b.z, x.b.w};
#pragma unroll
      for (int u = 0; u < UPT; ++u) {
        uint32_t o[4] = {0u, 0u, 0u, 0u}, r[4] = {0u, 0u, 0u, 0u};
        if (x.ok == 1) dequant_word<LO>(wd[u], u < 4 ? s_lo : s_hi, o, r);
        sts128(chunk_base + swz(trow, unit0 + u), o[0], o[1], o[2], o[3]);
        if constexpr (LO) sts128(chunk_base + NTL * 128 + swz(trow, unit0 + u), r[0], r[1], r[2], r[3]);
      }
    };
    auto process = [&](int j, const Raw& x) -> bool {
      const int b = j % NS, u = j / NS;
      if (x.ok == 2 && slot == 0 && kvh == 0 && (((st0 + j) * NT + tk) & (p.block - 1)) == 0)
        flag(p.status, QKV_DEV_BAD_PAGE);
      if (is_k) {
        if (u >= 1 && !wait_bar(&bars.kfree[b], (uint32_t)(u - 1) & 1u, abort)) return false;
        put(s_base + K_OFF + b * (2 * KT) + chunk * (2 * NTL * 128), x, std::true_type{});
        fence_async_smem();
        arrive_rank0(&bars.kready[b]);
      } else {
        if (u >= 1 && !wait_bar(&bars.vfree[b], (uint32_t)(u - 1) & 1u, abort)) return false;
        put(s_base + V_OFF + b * VT + chunk * (NT * 128), x, std::false_type{});
        fence_async_smem();
        arrive_rank0(&bars.vready[b]);
      }
      return true;
    };
    Raw ra, rb;
    ra.page = page_of(0);
    rb.page = page_of(1);
    load(0, ra);
    load(1, rb);
    bool ok = true;
    for (int j = 0; j < n_st; j += 2) {
      if (!process(j, ra)) { ok = false; break; }
      load(j + 2, ra);
      if (j + 1 < n_st) {
        if (!process(j + 1, rb)) { ok = false; break; }
        load(j + 3, rb);
      }
    }
    if (!ok) {
      abort_pair(&bars.abort);
      flag(p.status, QKV_DEV_TIMEOUT);
    }
  }

  tc_fence_before();
  cluster_sync();  // every role of both CTAs is done with tensor memory
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
  }
}

}  // namespace prefill
}  // namespace qkv

using namespace qkv;

extern "C" size_t qkv_paged_prefill_workspace_bytes(int32_t n_q, int32_t q_heads, int32_t head_dim,
                                                   int32_t num_splits) {
  if (n_q < 0 || q_heads < 1 || head_dim < 1 || num_splits < 1) return 0;
  if (num_splits == 1) return 0;
  const size_t rows = (size_t)n_q * q_heads;
  const size_t o = (rows * num_splits * head_dim * 4 + 255) & ~size_t(255);
  const size_t l = (rows * num_splits * 4 + 255) & ~size_t(255);
  return o + l;
}

namespace qkv {

// The automatic part count: the fewest parts (at most max_parts and the
// stage count of the shortest pair) that fill the waves of CTA pairs (one
// CTA per SM) to 95 %. -1 when the device cannot be queried.
static int prefill_auto_parts(int pairs, int min_stages, int max_parts) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  const int slots = sms / 2 > 0 ? sms / 2 : 1;
  int S = 1;
  double best = 0.0;
  for (int c = 1; c <= max_parts && c <= min_stages; ++c) {
    const int units = pairs * c, waves = (units + slots - 1) / slots;
    const double eff = (double)units / ((double)waves * slots);
    if (eff > best + 1e-9) {
      best = eff;
      S = c;
    }
    if (eff >= 0.95) break;
  }
  return S;
}

// Validation and launch of the prefill kernel. Query i of the chunk attends
// tokens 0 .. min(prefix_len + i, kv_limit - 1) of the page-table row.
// num_splits 0: automatic, at most max_parts parts. With o_part set, every
// part writes its fp32 partial and lse2 to o_part / lse_part [part][n_q *
// q_heads] (the caller merges); without, num_splits must come out 1 and the
// kernel writes out and lse2 itself. *parts_used gets the part count.
int prefill_run(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
                const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, int32_t n_q,
                int32_t prefix_len, int32_t kv_limit, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                int32_t v_group, int32_t num_splits, int32_t max_parts, float* o_part, float* lse_part,
                int32_t* device_status, cudaStream_t stream, int* parts_used) {
  if (!q || !k_data || !k_scale || !v_data || !v_scale || !page_table || (!o_part && !out)) return QKV_EINVAL;
  if (n_q < 0 || prefix_len < 0 || kv_limit < 1 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads ||
      block_size < 1 || max_pages_per_seq < 1 || num_pages < 1 || !(softmax_scale >= 0.f) ||
      !isfinite(softmax_scale) || (v_group != 32 && v_group != head_dim) || num_splits < 0 || num_splits > 64 ||
      max_parts < 1)
    return QKV_EINVAL;
  const int64_t span = std::min<int64_t>((int64_t)prefix_len + n_q, kv_limit);
  if (span > (int64_t)max_pages_per_seq * block_size) return QKV_EINVAL;
  if (((uintptr_t)out | (uintptr_t)q | (uintptr_t)k_data | (uintptr_t)v_data | (uintptr_t)o_part) & 15)
    return QKV_EINVAL;
  if (((uintptr_t)k_scale | (uintptr_t)v_scale | (uintptr_t)lse2_out | (uintptr_t)lse_part) & 3) return QKV_EINVAL;
  if (o_part && !lse_part) return QKV_EINVAL;
  const int G = q_heads / kv_heads;
  if ((head_dim != 256 && head_dim != 128) || (G != 1 && G != 2 && G != 4 && G != 8)) return QKV_EUNSUPPORTED;
  if (block_size & (block_size - 1)) return QKV_EUNSUPPORTED;  // pages of a power-of-two size
  if (kv_heads > 65535) return QKV_EUNSUPPORTED;
  if (n_q == 0) {
    *parts_used = 0;
    return QKV_OK;
  }

  const int QB = prefill::M / G;
  const int pairs_x = (n_q + QB - 1) / QB;
  // the smallest context of a pair (the first query block) bounds the parts
  const int64_t first_span = std::min<int64_t>((int64_t)prefix_len + (n_q < QB ? n_q : QB), kv_limit);
  const int min_stages = (int)((first_span + prefill::NT - 1) / prefill::NT);
  int S = num_splits;
  if (S == 0) {
    S = prefill_auto_parts(pairs_x * kv_heads, min_stages, max_parts);
    if (S < 0) return QKV_ECUDA;
  }
  if (S > min_stages || S > max_parts) return QKV_EINVAL;  // a part without a stage, or no room for it
  if (!o_part && S != 1) return QKV_EINVAL;

  prefill::Params p;
  p.q = q;
  p.out = out;
  p.lse2 = lse2_out;
  p.k_data = k_data;
  p.k_scale = k_scale;
  p.v_data = v_data;
  p.v_scale = v_scale;
  p.page_table = page_table;
  p.num_pages = num_pages;
  p.n_q = n_q;
  p.prefix_len = prefix_len;
  p.kv_limit = kv_limit;
  p.q_heads = q_heads;
  p.kv_heads = kv_heads;
  p.G = G;
  p.QB = QB;
  p.block = block_size;
  p.block_shift = 0;
  while ((1 << p.block_shift) < block_size) ++p.block_shift;
  p.v_tok = v_group != 32;
  const float sc = softmax_scale > 0.f ? softmax_scale : 1.f / sqrtf((float)head_dim);
  p.score_scale = sc * 1.4426950408889634f;
  p.status = device_status;
  p.n_splits = S;
  p.o_part = o_part;
  p.lse_part = lse_part;

  const bool d128 = head_dim == 128;
  const void* fn = d128 ? (const void*)prefill::paged_prefill_kernel<128> : (const void*)prefill::paged_prefill_kernel<256>;
  const int smem = d128 ? prefill::Geo<128>::SMEM_BYTES : prefill::Geo<256>::SMEM_BYTES;
  static bool attr_set[64][2];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QKV_ECUDA;
  if (!attr_set[dev][d128]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
      (void)cudaGetLastError();
      return QKV_ECUDA;
    }
    attr_set[dev][d128] = true;
  }
  // one CTA pair (a cluster of two, compiled in) per (256 / G queries, KV head, part)
  const dim3 grid(2u * (unsigned)pairs_x, (unsigned)kv_heads, (unsigned)S);
  void* args[] = {&p};
  if (launch_pdl(fn, grid, dim3(prefill::THREADS), smem, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  *parts_used = S;
  return QKV_OK;
}

// Parts the one-call entry may use within workspace_bytes (at most 8).
static int prefill_max_parts(int32_t n_q, int32_t q_heads, int32_t head_dim, size_t workspace_bytes) {
  int c = 1;
  while (c < 8 && workspace_bytes >= qkv_paged_prefill_workspace_bytes(n_q, q_heads, head_dim, c + 1)) ++c;
  return c;
}

}  // namespace qkv

extern "C" int32_t qkv_paged_prefill_auto_splits(int32_t n_q, int32_t prefix_len, int32_t q_heads,
                                                 int32_t kv_heads, int32_t head_dim, size_t workspace_bytes) {
  if (n_q < 1 || prefix_len < 0 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads ||
      (head_dim != 256 && head_dim != 128))
    return 0;
  const int G = q_heads / kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
  const int QB = prefill::M / G;
  const int min_stages = (prefix_len + (n_q < QB ? n_q : QB) + prefill::NT - 1) / prefill::NT;
  const int S = prefill_auto_parts((n_q + QB - 1) / QB * kv_heads, min_stages,
                                   prefill_max_parts(n_q, q_heads, head_dim, workspace_bytes));
  return S < 0 ? 0 : S;
}

extern "C" int qkv_paged_prefill_attn_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                                         const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                         const int32_t* page_table, int32_t n_q, int32_t prefix_len,
                                         int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                         int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                         int32_t v_group, int32_t num_splits, void* workspace,
                                         size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream) {
  if (n_q == 0) return QKV_OK;
  if (!out) return QKV_EINVAL;
  if ((uintptr_t)workspace & 255) return QKV_EINVAL;
  if (n_q < 0 || q_heads < 1 || head_dim < 1) return QKV_EINVAL;
  const int max_parts = prefill_max_parts(n_q, q_heads, head_dim, workspace ? workspace_bytes : 0);
  if (num_splits > 1 && (!workspace || workspace_bytes < qkv_paged_prefill_workspace_bytes(n_q, q_heads, head_dim,
                                                                                            num_splits)))
    return QKV_EINVAL;
  const int cap = num_splits > 0 ? num_splits : max_parts;
  // run as one part unless the plan splits; a split run writes partials into the workspace
  const size_t rows = (size_t)n_q * q_heads;
  float* o_part = reinterpret_cast<float*>(workspace);
  float* lse_part = workspace ? reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                                          ((rows * cap * head_dim * 4 + 255) & ~size_t(255)))
                              : nullptr;
  int S = num_splits;
  if (S == 0) {
    S = qkv_paged_prefill_auto_splits(n_q, prefix_len, q_heads, kv_heads, head_dim, workspace ? workspace_bytes : 0);
    if (S < 1) S = 1;  // invalid shapes are reported by the run below
  }
  int used = 0;
  const int rc = prefill_run(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, n_q, prefix_len,
                             0x7fffffff, q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages,
                             softmax_scale, v_group, S, S > 1 ? cap : 1, S > 1 ? o_part : nullptr,
                             S > 1 ? lse_part : nullptr, device_status, stream, &used);
  if (rc || used <= 1) return rc;
  return qkv_lse_merge(o_part, lse_part, used, (int32_t)rows, head_dim, out, lse2_out, stream);
}
