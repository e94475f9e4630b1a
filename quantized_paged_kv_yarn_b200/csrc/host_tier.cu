// host_tier.cu -- the host-placed K/V tier (sm_100a): pages of an F4 pool
// held in pinned host memory, streamed over the host link into a window of
// device pages, attended there by the split pass and folded with the
// log2-sum-exp merge.
//
// Source: "Serving Qwen3.8-Flash-Next's 1M-token window on one 24 GB card
// #568", Proposed solution, item 2 (host-placed K/V): the K/V of a long
// context lives in host RAM, decode reads it over PCIe, a prefill stages its
// pages into a 131,072-token device window, and the windows' partial results
// are folded by log2-sum-exp.
//
// B200 design: the tier's bytes cross the host link exactly once per step in
// either form, so the kernel that reads host memory is a plain gather (16-byte
// loads of mapped pinned memory, many in flight per SM) into a device window,
// and the attention over the window is the TMA-fed split kernel reading HBM
// at ~4.6 TB/s -- about 1 % of the link time of the same bytes.
#include "common.cuh"

#include <algorithm>

namespace qkv {

// The four arrays of a pool (K data, K scales, V data, V scales), each a
// slab of a fixed number of 16-byte units per page.
struct StageParams {
  const uint4* src[4];
  uint4* dst[4];
  int64_t slab[4];  // 16-byte units per page
  const int32_t* src_pages;
  int64_t src_num_pages;
  int64_t dst_page0;
  int32_t* status;
  int32_t* tab_out;  // nullable: tab_out[i] = i for i < n_pages (the window's page table)
  int32_t* len_out;  // nullable: *len_out = len_value (the window's token count)
  int32_t len_value;
  int32_t n_pages;
};

constexpr int STAGE_THREADS = 256;
constexpr int STAGE_UNROLL = 4;  // loads in flight per thread before its stores

// A persistent grid of one CTA per SM at most (256 threads, no shared
// memory). Each CTA walks destination pages i = blockIdx.x, + gridDim.x, ...:
// the source page id is read once, then each array's slab is copied with
// STAGE_UNROLL independent 16-byte loads per thread ahead of the stores (the
// link's latency is microseconds; a few MB in flight across the grid keep it
// busy).
//
// Unlike the other kernels it does not let its successor start early: the
// attention kernels that follow it would otherwise sit on the same SMs while
// its loads of host memory are outstanding. (With a prefill kernel running
// beside a live staging grid -- staging on a second stream -- a bounded wait
// of the prefill ran out at full size, both before and after the prefill
// took its tensor memory only after its dependency wait. A race found later
// fits it: the prefill's one P-ready barrier let a CTA running a stage ahead
// of its partner complete the partner's phase, after which the partner
// could wait for scores that never came; a staging CTA on one SM of a pair
// is what slows one CTA of it. That barrier is now split by stage parity,
// but the overlap has not been run since, so the library still never
// overlaps the two.)
__global__ void __launch_bounds__(STAGE_THREADS) stage_pages_f4_kernel(const StageParams p) {
  pdl_wait();
  if (blockIdx.x == 0) {
    if (p.tab_out)
      for (int j = threadIdx.x; j < p.n_pages; j += STAGE_THREADS) p.tab_out[j] = j;
    if (p.len_out && threadIdx.x == 0) *p.len_out = p.len_value;
  }
#pragma unroll 1
  for (int i = blockIdx.x; i < p.n_pages; i += gridDim.x) {
    const int32_t page = p.src_pages[i];
    const bool bad = page < 0 || page >= p.src_num_pages;
    if (bad && threadIdx.x == 0) flag(p.status, QKV_DEV_BAD_PAGE);
#pragma unroll 1
    for (int a = 0; a < 4; ++a) {
      const int64_t n = p.slab[a];
      uint4* d = p.dst[a] + (p.dst_page0 + i) * n;
      if (bad) {
        for (int64_t u = threadIdx.x; u < n; u += STAGE_THREADS) d[u] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const uint4* s = p.src[a] + (int64_t)page * n;
#pragma unroll 1
      for (int64_t u0 = threadIdx.x; u0 < n; u0 += STAGE_THREADS * STAGE_UNROLL) {
        uint4 v[STAGE_UNROLL];
#pragma unroll
        for (int k = 0; k < STAGE_UNROLL; ++k) {
          const int64_t u = u0 + (int64_t)k * STAGE_THREADS;
          if (u < n) v[k] = s[u];
        }
#pragma unroll
        for (int k = 0; k < STAGE_UNROLL; ++k) {
          const int64_t u = u0 + (int64_t)k * STAGE_THREADS;
          if (u < n) d[u] = v[k];
        }
      }
    }
  }
}

// The address a kernel on the current device uses for `p`: device and managed
// memory as they are, pinned host memory through its mapping. Pageable host
// memory (or an address no allocation covers) has none.
bool device_view(const void* p, const void** dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  switch (a.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
      *dev = p;
      return true;
    case cudaMemoryTypeHost:
      *dev = a.devicePointer;
      return a.devicePointer != nullptr;
    default:
      return false;
  }
}

struct Slabs {
  int64_t bytes[4];  // K data, K scales, V data, V scales per page
};

bool slabs_of(int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t v_group, Slabs& s) {
  if (kv_heads < 1 || head_dim < 32 || head_dim > 256 || head_dim % 32 || block_size < 1 || block_size > 1024 ||
      (v_group != 32 && v_group != head_dim))
    return false;
  const int64_t rows = (int64_t)kv_heads * block_size;
  s.bytes[0] = s.bytes[2] = rows * (head_dim / 2);
  s.bytes[1] = rows * (head_dim / 32) * 2;
  s.bytes[3] = rows * (head_dim / v_group) * 2;
  for (int a = 0; a < 4; ++a)
    if (s.bytes[a] % 16) return false;  // 16-byte units (kv_heads * block_size even enough)
  return true;
}

int stage_impl(void* const dst[4], int64_t dst_num_pages, int64_t dst_page0, const void* const src[4],
               int64_t src_num_pages, const int32_t* src_pages, int32_t n_pages, const Slabs& sl,
               int32_t* tab_out, int32_t* len_out, int32_t len_value, int32_t* status, cudaStream_t stream) {
  if (n_pages == 0) return QKV_OK;
  StageParams p;
  for (int a = 0; a < 4; ++a) {
    p.src[a] = reinterpret_cast<const uint4*>(src[a]);
    p.dst[a] = reinterpret_cast<uint4*>(dst[a]);
    p.slab[a] = sl.bytes[a] / 16;
  }
  p.src_pages = src_pages;
  p.src_num_pages = src_num_pages;
  p.dst_page0 = dst_page0;
  p.status = status;
  p.tab_out = tab_out;
  p.len_out = len_out;
  p.len_value = len_value;
  p.n_pages = n_pages;
  (void)dst_num_pages;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess || sms < 1) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  void* args[] = {&p};
  if (launch_pdl((const void*)stage_pages_f4_kernel, dim3((unsigned)std::min(n_pages, sms)), dim3(STAGE_THREADS), 0,
                 stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the tiered decode: the window (four page arrays), its page
// table and token count, then the partials of one sequence.
struct TierLayout {
  size_t win[4], tab, len, o, lse, total;
  int64_t parts;
};

bool tier_layout(int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t v_group,
                 int32_t max_host_pages_per_seq, int32_t window_pages, int32_t max_splits, TierLayout& L) {
  Slabs sl;
  if (q_heads < 1 || max_host_pages_per_seq < 0 || window_pages < 1 || max_splits < 1 ||
      !slabs_of(kv_heads, head_dim, block_size, v_group, sl))
    return false;
  size_t off = 0;
  for (int a = 0; a < 4; ++a) {
    L.win[a] = off;
    off += align256((size_t)window_pages * sl.bytes[a]);
  }
  L.tab = off;
  off += align256((size_t)window_pages * 4);
  L.len = off;
  off += 256;
  const int64_t windows = ((int64_t)max_host_pages_per_seq + window_pages - 1) / window_pages;
  L.parts = (windows + 1) * max_splits;
  L.o = off;
  off += align256((size_t)L.parts * q_heads * head_dim * 4);
  L.lse = off;
  off += align256((size_t)L.parts * q_heads * 4);
  L.total = off;
  return true;
}

// Prefill kernel run (prefill.cu): query i attends tokens
// 0 .. min(prefix_len + i, kv_limit - 1); with o_part every part writes its
// fp32 partial for the caller's merge.
int prefill_run(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
                const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, int32_t n_q,
                int32_t prefix_len, int32_t kv_limit, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                int32_t v_group, int32_t num_splits, int32_t max_parts, float* o_part, float* lse_part,
                int32_t* device_status, cudaStream_t stream, int* parts_used);

// Workspace of the tiered prefill: the window and its page table, then the
// fp32 partials of every part of every window and of the device part.
bool prefill_tier_layout(int32_t n_q, int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                         int32_t v_group, int32_t max_host_pages, int32_t window_pages, int32_t parts_per_launch,
                         TierLayout& L) {
  Slabs sl;
  if (n_q < 1 || q_heads < 1 || max_host_pages < 0 || window_pages < 1 || parts_per_launch < 1 ||
      parts_per_launch > 64 || !slabs_of(kv_heads, head_dim, block_size, v_group, sl))
    return false;
  size_t off = 0;
  for (int a = 0; a < 4; ++a) {
    L.win[a] = off;
    off += align256((size_t)window_pages * sl.bytes[a]);
  }
  L.tab = off;
  off += align256((size_t)window_pages * 4);
  L.len = off;
  off += 256;
  const int64_t windows = ((int64_t)max_host_pages + window_pages - 1) / window_pages;
  L.parts = (windows + 1) * parts_per_launch;
  const size_t rows = (size_t)n_q * q_heads;
  L.o = off;
  off += align256((size_t)L.parts * rows * head_dim * 4);
  L.lse = off;
  off += align256((size_t)L.parts * rows * 4);
  L.total = off;
  return true;
}

}  // namespace qkv

using namespace qkv;

extern "C" int qkv_stage_pages_f4(uint8_t* dst_k_data, uint16_t* dst_k_scale, uint8_t* dst_v_data,
                                  uint16_t* dst_v_scale, int64_t dst_num_pages, int64_t dst_page0,
                                  const uint8_t* src_k_data, const uint16_t* src_k_scale, const uint8_t* src_v_data,
                                  const uint16_t* src_v_scale, int64_t src_num_pages, const int32_t* src_pages,
                                  int32_t n_pages, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t v_group, int32_t* device_status, qkv_stream_t stream) {
  Slabs sl;
  if (!slabs_of(kv_heads, head_dim, block_size, v_group, sl)) return QKV_EINVAL;
  if (n_pages < 0 || dst_num_pages < 1 || src_num_pages < 1 || dst_page0 < 0 ||
      dst_page0 + n_pages > dst_num_pages)
    return QKV_EINVAL;
  if (n_pages == 0) return QKV_OK;
  void* dst[4] = {dst_k_data, dst_k_scale, dst_v_data, dst_v_scale};
  const void* src_host[4] = {src_k_data, src_k_scale, src_v_data, src_v_scale};
  const void* src[4];
  const void* pages = nullptr;
  for (int a = 0; a < 4; ++a) {
    if (!dst[a] || !src_host[a] || ((uintptr_t)dst[a] & 15) || ((uintptr_t)src_host[a] & 15)) return QKV_EINVAL;
    if (!device_view(src_host[a], &src[a])) return QKV_EINVAL;
  }
  if (!src_pages || ((uintptr_t)src_pages & 3) || !device_view(src_pages, &pages)) return QKV_EINVAL;
  return stage_impl(dst, dst_num_pages, dst_page0, src, src_num_pages, static_cast<const int32_t*>(pages), n_pages,
                    sl, nullptr, nullptr, 0, device_status, stream);
}

extern "C" size_t qkv_paged_decode_tiered_workspace_bytes(int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                                          int32_t block_size, int32_t v_group,
                                                          int32_t max_host_pages_per_seq, int32_t window_pages,
                                                          int32_t max_splits) {
  TierLayout L;
  if (!tier_layout(q_heads, kv_heads, head_dim, block_size, v_group, max_host_pages_per_seq, window_pages,
                   max_splits, L))
    return 0;
  return L.total;
}

extern "C" int qkv_paged_decode_attn_f4_tiered(
    uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
    const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, const int32_t* seq_lens,
    int32_t max_pages_per_seq, int64_t num_pages, const uint8_t* host_k_data, const uint16_t* host_k_scale,
    const uint8_t* host_v_data, const uint16_t* host_v_scale, int64_t host_num_pages,
    const int32_t* host_page_table, int32_t max_host_pages_per_seq, const int32_t* host_lens, int32_t n_seq,
    int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t v_group, float softmax_scale,
    int32_t window_pages, int32_t max_splits, void* workspace, size_t workspace_bytes, int32_t* device_status,
    qkv_stream_t stream) {
  if (n_seq < 0) return QKV_EINVAL;
  if (n_seq == 0) return QKV_OK;
  if (!out || !q || !k_data || !k_scale || !v_data || !v_scale || !page_table || !seq_lens || !host_k_data ||
      !host_k_scale || !host_v_data || !host_v_scale || !host_page_table || !host_lens || !workspace)
    return QKV_EINVAL;
  if (max_pages_per_seq < 1 || num_pages < 1 || host_num_pages < 1 || max_host_pages_per_seq < 1 ||
      q_heads < 1 || kv_heads < 1 || q_heads % kv_heads || ((uintptr_t)workspace & 255))
    return QKV_EINVAL;
  TierLayout L;
  if (!tier_layout(q_heads, kv_heads, head_dim, block_size, v_group, max_host_pages_per_seq, window_pages,
                   max_splits, L) ||
      workspace_bytes < L.total)
    return QKV_EINVAL;
  if ((int64_t)window_pages * block_size > 0x7fffffffLL) return QKV_EUNSUPPORTED;
  // host_lens is host memory: every length is checked before the first launch
  for (int s = 0; s < n_seq; ++s)
    if (host_lens[s] < 0 || host_lens[s] % block_size || host_lens[s] / block_size > max_host_pages_per_seq)
      return QKV_EINVAL;
  const void* src_host[4] = {host_k_data, host_k_scale, host_v_data, host_v_scale};
  const void* src[4];
  for (int a = 0; a < 4; ++a)
    if (((uintptr_t)src_host[a] & 15) || !device_view(src_host[a], &src[a])) return QKV_EINVAL;
  const void* hpt;
  if (((uintptr_t)host_page_table & 3) || !device_view(host_page_table, &hpt)) return QKV_EINVAL;
  const int32_t* host_pt = static_cast<const int32_t*>(hpt);

  char* ws = static_cast<char*>(workspace);
  void* win[4];
  for (int a = 0; a < 4; ++a) win[a] = ws + L.win[a];
  int32_t* tab = reinterpret_cast<int32_t*>(ws + L.tab);
  int32_t* len = reinterpret_cast<int32_t*>(ws + L.len);
  float* o = reinterpret_cast<float*>(ws + L.o);
  float* lse = reinterpret_cast<float*>(ws + L.lse);
  Slabs sl;
  slabs_of(kv_heads, head_dim, block_size, v_group, sl);
  const size_t qrow = (size_t)q_heads * head_dim;

  for (int s = 0; s < n_seq; ++s) {
    const int32_t n_host = host_lens[s] / block_size;
    int64_t parts = 0;
    // the host part, one window at a time
    for (int32_t c0 = 0; c0 < n_host; c0 += window_pages) {
      const int32_t n = std::min(window_pages, n_host - c0);
      int rc = stage_impl(win, window_pages, 0, src, host_num_pages,
                          host_pt + (size_t)s * max_host_pages_per_seq + c0, n, sl, tab, len, n * block_size,
                          device_status, stream);
      if (rc) return rc;
      rc = qkv_paged_decode_split_f4_v(o + (size_t)parts * qrow, lse + (size_t)parts * q_heads, max_splits,
                                       q + s * qrow, static_cast<const uint8_t*>(win[0]),
                                       static_cast<const uint16_t*>(win[1]), static_cast<const uint8_t*>(win[2]),
                                       static_cast<const uint16_t*>(win[3]), tab, len, 1, q_heads, kv_heads,
                                       head_dim, block_size, window_pages, window_pages, softmax_scale, 0, v_group,
                                       device_status, stream);
      if (rc) return rc;
      parts += max_splits;
    }
    // the device part
    int rc = qkv_paged_decode_split_f4_v(o + (size_t)parts * qrow, lse + (size_t)parts * q_heads, max_splits,
                                         q + s * qrow, k_data, k_scale, v_data, v_scale,
                                         page_table + (size_t)s * max_pages_per_seq, seq_lens + s, 1, q_heads,
                                         kv_heads, head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale,
                                         0, v_group, device_status, stream);
    if (rc) return rc;
    parts += max_splits;
    rc = qkv_lse_merge(o, lse, (int32_t)parts, q_heads, head_dim, out + s * qrow,
                       lse2_out ? lse2_out + (size_t)s * q_heads : nullptr, stream);
    if (rc) return rc;
  }
  return QKV_OK;
}

extern "C" size_t qkv_paged_prefill_tiered_workspace_bytes(int32_t n_q, int32_t q_heads, int32_t kv_heads,
                                                           int32_t head_dim, int32_t block_size, int32_t v_group,
                                                           int32_t max_host_pages, int32_t window_pages,
                                                           int32_t parts_per_launch) {
  TierLayout L;
  if (!prefill_tier_layout(n_q, q_heads, kv_heads, head_dim, block_size, v_group, max_host_pages, window_pages,
                           parts_per_launch, L))
    return 0;
  return L.total;
}

extern "C" int qkv_paged_prefill_attn_f4_tiered(
    uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
    const uint8_t* v_data, const uint16_t* v_scale, const int32_t* page_table, int32_t n_q, int32_t prefix_len,
    int32_t max_pages_per_seq, int64_t num_pages, const uint8_t* host_k_data, const uint16_t* host_k_scale,
    const uint8_t* host_v_data, const uint16_t* host_v_scale, int64_t host_num_pages,
    const int32_t* host_page_table, int32_t host_len, int32_t q_heads, int32_t kv_heads, int32_t head_dim,
    int32_t block_size, int32_t v_group, float softmax_scale, int32_t window_pages, int32_t parts_per_launch,
    void* workspace, size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream) {
  if (n_q == 0) return QKV_OK;
  if (!out || !q || !host_k_data || !host_k_scale || !host_v_data || !host_v_scale || !host_page_table ||
      !workspace || n_q < 0 || host_len < 0 || host_num_pages < 1 || block_size < 1 || host_len % block_size ||
      ((uintptr_t)workspace & 255))
    return QKV_EINVAL;
  const int32_t n_host = host_len / block_size;
  TierLayout L;
  if (!prefill_tier_layout(n_q, q_heads, kv_heads, head_dim, block_size, v_group, n_host, window_pages,
                           parts_per_launch, L) ||
      workspace_bytes < L.total)
    return QKV_EINVAL;
  if ((int64_t)window_pages * block_size > 0x7fffffffLL) return QKV_EUNSUPPORTED;
  const void* src_host[4] = {host_k_data, host_k_scale, host_v_data, host_v_scale};
  const void* src[4];
  for (int a = 0; a < 4; ++a)
    if (((uintptr_t)src_host[a] & 15) || !device_view(src_host[a], &src[a])) return QKV_EINVAL;
  const void* hpt;
  if (((uintptr_t)host_page_table & 3) || !device_view(host_page_table, &hpt)) return QKV_EINVAL;

  char* ws = static_cast<char*>(workspace);
  void* win[4];
  for (int a = 0; a < 4; ++a) win[a] = ws + L.win[a];
  int32_t* tab = reinterpret_cast<int32_t*>(ws + L.tab);
  float* o = reinterpret_cast<float*>(ws + L.o);
  float* lse = reinterpret_cast<float*>(ws + L.lse);
  Slabs sl;
  slabs_of(kv_heads, head_dim, block_size, v_group, sl);
  const size_t rows = (size_t)n_q * q_heads;

  int64_t parts = 0;
  int used = 0;
  for (int32_t c0 = 0; c0 < n_host; c0 += window_pages) {
    const int32_t n = std::min(window_pages, n_host - c0);
    int rc = stage_impl(win, window_pages, 0, src, host_num_pages, static_cast<const int32_t*>(hpt) + c0, n, sl, tab,
                        nullptr, 0, device_status, stream);
    if (rc) return rc;
    // every query of the chunk sees every token of the window
    rc = prefill_run(out, nullptr, q, static_cast<const uint8_t*>(win[0]), static_cast<const uint16_t*>(win[1]),
                     static_cast<const uint8_t*>(win[2]), static_cast<const uint16_t*>(win[3]), tab, n_q,
                     n * block_size, n * block_size, q_heads, kv_heads, head_dim, block_size, window_pages,
                     window_pages, softmax_scale, v_group, 0, parts_per_launch, o + (size_t)parts * rows * head_dim,
                     lse + (size_t)parts * rows, device_status, stream, &used);
    if (rc) return rc;
    parts += used;
  }
  // the device part: causal over the device tokens, the chunk at prefix_len ..
  int rc = prefill_run(out, nullptr, q, k_data, k_scale, v_data, v_scale, page_table, n_q, prefix_len, 0x7fffffff,
                       q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale, v_group, 0,
                       parts_per_launch, o + (size_t)parts * rows * head_dim, lse + (size_t)parts * rows,
                       device_status, stream, &used);
  if (rc) return rc;
  parts += used;
  return qkv_lse_merge(o, lse, (int32_t)parts, (int32_t)rows, head_dim, out, lse2_out, stream);
}
