// decode_split.cu -- host side of the split pass of paged GQA decode
// attention over the F4 cache (kernel in decode_split.cuh), the one-call
// decode attention (split pass + log2-sum-exp merge) and the decode step.
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 2
// (v1/v2 paged attention that dequantises F4 cells inline; v2 partitions the
// context and reduces the partitions); FreeToken issue #568 "Serving ...'s
// 1M-token window on one 24 GB card", proposed solution item 2 (partials
// folded by log2-sum-exp).
#include "decode_split.cuh"

// ======================================================================= host side

namespace qkv {
extern template const void* split_kernel<128>(int, int, bool, bool);
extern template size_t split_kernel_smem<128>(int);
}  // namespace qkv

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

// 2-D view [rows][head_dim / 2 bytes] of a packed cache, boxes of `block`
// rows, the swizzle of the row width (128-byte rows: 128B, 64-byte rows: 64B).
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, int block, int head_dim) {
  EncodeTiled enc = encode_fn();
  if (!enc) return false;
  const int row_bytes = head_dim / 2;
  const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)block};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t kernel_smem(int head_dim, int G) {
  return head_dim == 128 ? split_kernel_smem<128>(G) : split_kernel_smem<256>(G);
}

const void* pick_kernel(int head_dim, int block, int G, bool vtok = false, bool fuse = false) {
  if (head_dim == 256) return split_kernel<256>(block, G, vtok, fuse);
  if (head_dim == 128) return split_kernel<128>(block, G, vtok, fuse);
  return nullptr;
}

constexpr int MAX_DEVICES = 64;

// Opt the kernel into its shared-memory size on the current device (once)
// and return its resident CTAs per SM.
int prepare(const void* fn, int head_dim, int block, int G, bool vtok = false, bool fuse = false) {
  static std::mutex mu;
  static int occ[MAX_DEVICES][2][3][4][4];  // [head_dim 128][block][G][vtok + 2 fuse]; 0 = not prepared
  const int vi = (vtok ? 1 : 0) + (fuse ? 2 : 0);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return 0;
  const int di = head_dim == 128 ? 1 : 0;
  const int bi = block == 16 ? 0 : block == 32 ? 1 : 2;
  const int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  std::lock_guard<std::mutex> lock(mu);
  if (occ[dev][di][bi][gi][vi] == 0) {
    const size_t smem = kernel_smem(head_dim, G);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, THREADS, smem) != cudaSuccess || n < 1)
      return 0;
    occ[dev][di][bi][gi][vi] = n;
  }
  return occ[dev][di][bi][gi][vi];
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
  const void* fn = pick_kernel(256, block_size, 4);
  if (!fn) return 0;
  const int occ = prepare(fn, 256, block_size, 4);
  const int sms = sm_count();
  if (occ < 1 || sms < 1) return 0;
  return (int32_t)std::max(1, occ * sms / kv_heads);
}

// Workspace of the one-call decode attention: o_parts, then lse2_parts from
// the next 256-byte boundary.
struct DecodeWs {
  size_t o, lse, total;
};
DecodeWs decode_ws(int64_t n_seq, int64_t q_heads, int64_t head_dim, int64_t max_splits) {
  const size_t rows = (size_t)n_seq * q_heads;
  DecodeWs w;
  w.o = 0;
  w.lse = (rows * max_splits * head_dim * 4 + 255) & ~size_t(255);
  w.total = w.lse + ((rows * max_splits * 4 + 255) & ~size_t(255));
  return w;
}

extern "C" size_t qkv_paged_decode_workspace_bytes(int32_t n_seq, int32_t q_heads, int32_t head_dim,
                                                   int32_t max_splits) {
  if (n_seq < 0 || q_heads < 0 || head_dim < 0 || max_splits < 0) return 0;
  return decode_ws(n_seq, q_heads, head_dim, max_splits).total;
}

// The decode step's inputs of the fused launch (qkv_decode_step_f4).
struct StepArgs {
  const uint16_t* k_new;
  const uint16_t* v_new;
  const int64_t* positions;
  const int64_t* slots;
  const float* cos_tab;
  const float* sin_tab;
  int64_t tab_start, tab_len;
  int rot;
};

static int split_impl(float* o_parts, float* lse2_parts, int32_t max_splits, const uint16_t* q,
                      const uint8_t* k_data, const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                      const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq, int32_t q_heads,
                      int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t max_pages_per_seq,
                      int64_t num_pages, float softmax_scale, int32_t num_splits, int32_t v_group,
                      int32_t* device_status, qkv_stream_t stream, const StepArgs* step) {
  if (!o_parts || !lse2_parts || !q || !k_data || !k_scale || !v_data || !v_scale || !page_table || !seq_lens)
    return QKV_EINVAL;
  if (n_seq < 0 || q_heads < 1 || kv_heads < 1 || max_pages_per_seq < 1 || num_pages < 1 || max_splits < 1 ||
      num_splits < 0 || num_splits > max_splits || block_size < 1 || !(softmax_scale >= 0.f) ||
      !isfinite(softmax_scale) ||
      (v_group != 32 && v_group != head_dim))
    return QKV_EINVAL;
  if (q_heads % kv_heads) return QKV_EINVAL;
  if (!aligned16(q) || !aligned16(k_data) || !aligned16(v_data) || !aligned16(k_scale) || !aligned16(v_scale) ||
      !aligned16(o_parts) || ((uintptr_t)lse2_parts & 3))
    return QKV_EINVAL;
  const int G = q_heads / kv_heads;
  if (head_dim != 256 && head_dim != 128) return QKV_EUNSUPPORTED;
  const bool vtok = v_group != 32;
  const void* fn = pick_kernel(head_dim, block_size, G, vtok, step != nullptr);
  if (!fn) return QKV_EUNSUPPORTED;
  const uint64_t cache_rows = (uint64_t)num_pages * kv_heads * block_size;
  if (cache_rows > 0x7fffffffull) return QKV_EUNSUPPORTED;  // TMA row coordinate is int32
  if ((int64_t)max_pages_per_seq * block_size > 0x7fffffffLL) return QKV_EUNSUPPORTED;
  if (max_splits > 65535 || n_seq > 65535 || kv_heads > 65535) return QKV_EUNSUPPORTED;
  if (n_seq == 0) return QKV_OK;

  const int occ = prepare(fn, head_dim, block_size, G, vtok, step != nullptr);
  const int sms = sm_count();
  if (occ < 1 || sms < 1) return QKV_ECUDA;

  CUtensorMap tm_k, tm_v;
  if (!make_map(&tm_k, k_data, cache_rows, block_size, head_dim) ||
      !make_map(&tm_v, v_data, cache_rows, block_size, head_dim))
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
  KParams<true> pf;  // the fused instances' parameters: Params + the step's inputs
  static_cast<Params&>(pf) = p;
  if (step) {
    pf.st.rot = step->rot;
    pf.st.v_group = v_group;
    pf.st.k_new = step->k_new;
    pf.st.v_new = step->v_new;
    pf.st.positions = step->positions;
    pf.st.slots = step->slots;
    pf.st.cos_tab = step->cos_tab;
    pf.st.sin_tab = step->sin_tab;
    pf.st.tab_start = step->tab_start;
    pf.st.tab_len = step->tab_len;
    pf.st.k_data_w = const_cast<uint8_t*>(k_data);
    pf.st.v_data_w = const_cast<uint8_t*>(v_data);
    pf.st.k_scale_w = reinterpret_cast<__half*>(const_cast<uint16_t*>(k_scale));
    pf.st.v_scale_w = reinterpret_cast<__half*>(const_cast<uint16_t*>(v_scale));
  }

  // Slots past the plan's split count still get lse2 = -inf: the grid
  // covers every slot the merge reads.
  dim3 grid((unsigned)kv_heads, (unsigned)max_splits, (unsigned)n_seq);
  void* args[] = {(void*)&tm_k, (void*)&tm_v, step ? (void*)&pf : (void*)&p};
  if (launch_pdl(fn, grid, dim3(THREADS), kernel_smem(head_dim, G), stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" int qkv_paged_decode_split_f4_v(float* o_parts, float* lse2_parts, int32_t max_splits,
                                           const uint16_t* q, const uint8_t* k_data, const uint16_t* k_scale,
                                           const uint8_t* v_data, const uint16_t* v_scale,
                                           const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                           int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                           int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                           int32_t num_splits, int32_t v_group, int32_t* device_status,
                                           qkv_stream_t stream) {
  return split_impl(o_parts, lse2_parts, max_splits, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq,
                    q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale, num_splits,
                    v_group, device_status, stream, nullptr);
}

extern "C" int qkv_paged_decode_split_f4(float* o_parts, float* lse2_parts, int32_t max_splits, const uint16_t* q,
                                         const uint8_t* k_data, const uint16_t* k_scale, const uint8_t* v_data,
                                         const uint16_t* v_scale, const int32_t* page_table,
                                         const int32_t* seq_lens, int32_t n_seq, int32_t q_heads,
                                         int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                         int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                         int32_t num_splits, int32_t* device_status, qkv_stream_t stream) {
  return qkv_paged_decode_split_f4_v(o_parts, lse2_parts, max_splits, q, k_data, k_scale, v_data, v_scale,
                                     page_table, seq_lens, n_seq, q_heads, kv_heads, head_dim, block_size,
                                     max_pages_per_seq, num_pages, softmax_scale, num_splits, 32, device_status,
                                     stream);
}

// a4 + a5 (+ a2 + a3 with step): the split pass into the workspace, then
// the merge of its partials.
static int attn_impl(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                     const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                     const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq, int32_t q_heads,
                     int32_t kv_heads, int32_t head_dim, int32_t block_size, int32_t max_pages_per_seq,
                     int64_t num_pages, float softmax_scale, int32_t num_splits, int32_t max_splits, int32_t v_group,
                     void* workspace, size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream,
                     const StepArgs* step) {
  if (!out || !workspace) return QKV_EINVAL;
  if (((uintptr_t)workspace & 255) || max_splits < 1 || n_seq < 0 || q_heads < 1 || kv_heads < 1 ||
      head_dim < 1)
    return QKV_EINVAL;
  if (((uintptr_t)out & 3) || ((uintptr_t)lse2_out & 3)) return QKV_EINVAL;
  const DecodeWs L = decode_ws(n_seq, q_heads, head_dim, max_splits);
  if (workspace_bytes < L.total) return QKV_EINVAL;
  if (n_seq == 0) return QKV_OK;
  const size_t rows = (size_t)n_seq * q_heads;
  char* ws = static_cast<char*>(workspace);
  float* o_parts = reinterpret_cast<float*>(ws + L.o);
  float* lse_parts = reinterpret_cast<float*>(ws + L.lse);
  int rc = split_impl(o_parts, lse_parts, max_splits, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens,
                      n_seq, q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale,
                      num_splits, v_group, device_status, stream, step);
  if (rc != QKV_OK) return rc;
  return qkv_lse_merge(o_parts, lse_parts, max_splits, (int32_t)rows, head_dim, out, lse2_out, stream);
}

extern "C" int qkv_paged_decode_attn_f4_v(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                                          const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                          const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                          int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                          int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                          int32_t num_splits, int32_t max_splits, int32_t v_group, void* workspace,
                                          size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream) {
  return attn_impl(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq, q_heads, kv_heads,
                   head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale, num_splits, max_splits, v_group,
                   workspace, workspace_bytes, device_status, stream, nullptr);
}

extern "C" int qkv_decode_step_split_f4(float* o_parts, float* lse2_parts, int32_t max_splits, const uint16_t* q,
                                        const uint16_t* k_new, const uint16_t* v_new, const int64_t* positions,
                                        const int64_t* slot_mapping, const float* cos_tab, const float* sin_tab,
                                        int64_t table_pos_start, int64_t table_len, int32_t rot_dim,
                                        uint8_t* k_data, uint16_t* k_scale, uint8_t* v_data, uint16_t* v_scale,
                                        const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                        int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                        int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                        int32_t num_splits, int32_t v_group, int32_t* device_status,
                                        qkv_stream_t stream) {
  if (!k_new || !v_new || !positions || !slot_mapping || !cos_tab || !sin_tab) return QKV_EINVAL;
  if (rot_dim < 16 || rot_dim % 16 || rot_dim > head_dim || table_len < 0) return QKV_EINVAL;
  if (((uintptr_t)k_new | (uintptr_t)v_new) & 15) return QKV_EINVAL;
  const StepArgs step = {k_new, v_new, positions, slot_mapping, cos_tab, sin_tab, table_pos_start, table_len, rot_dim};
  return split_impl(o_parts, lse2_parts, max_splits, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq,
                    q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale, num_splits,
                    v_group, device_status, stream, &step);
}

extern "C" int qkv_decode_step_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint16_t* k_new,
                                  const uint16_t* v_new, const int64_t* positions, const int64_t* slot_mapping,
                                  const float* cos_tab, const float* sin_tab, int64_t table_pos_start,
                                  int64_t table_len, int32_t rot_dim, uint8_t* k_data, uint16_t* k_scale,
                                  uint8_t* v_data, uint16_t* v_scale, const int32_t* page_table,
                                  const int32_t* seq_lens, int32_t n_seq, int32_t q_heads, int32_t kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages,
                                  float softmax_scale, int32_t num_splits, int32_t max_splits, int32_t v_group,
                                  void* workspace, size_t workspace_bytes, int32_t* device_status,
                                  qkv_stream_t stream) {
  if (!k_new || !v_new || !positions || !slot_mapping || !cos_tab || !sin_tab) return QKV_EINVAL;
  if (rot_dim < 16 || rot_dim % 16 || rot_dim > head_dim || table_len < 0) return QKV_EINVAL;
  if (((uintptr_t)k_new | (uintptr_t)v_new) & 15) return QKV_EINVAL;
  const StepArgs step = {k_new, v_new, positions, slot_mapping, cos_tab, sin_tab, table_pos_start, table_len, rot_dim};
  return attn_impl(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq, q_heads, kv_heads,
                   head_dim, block_size, max_pages_per_seq, num_pages, softmax_scale, num_splits, max_splits, v_group,
                   workspace, workspace_bytes, device_status, stream, &step);
}

extern "C" int qkv_paged_decode_attn_f4(uint16_t* out, float* lse2_out, const uint16_t* q, const uint8_t* k_data,
                                        const uint16_t* k_scale, const uint8_t* v_data, const uint16_t* v_scale,
                                        const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                        int32_t q_heads, int32_t kv_heads, int32_t head_dim, int32_t block_size,
                                        int32_t max_pages_per_seq, int64_t num_pages, float softmax_scale,
                                        int32_t num_splits, int32_t max_splits, void* workspace,
                                        size_t workspace_bytes, int32_t* device_status, qkv_stream_t stream) {
  return qkv_paged_decode_attn_f4_v(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq,
                                    q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages,
                                    softmax_scale, num_splits, max_splits, 32, workspace, workspace_bytes,
                                    device_status, stream);
}
