// static_scratch.cu -- decode attention for callers that cannot allocate
// device memory.
//
// Some callers can't call cudaMalloc: plugins that run inside a host engine
// which owns every byte of device memory, and runtimes that plan their whole
// memory budget at start-up and forbid allocation afterwards (cudaMalloc can
// synchronise the device and fragments the planned budget). They cannot
// provide the partials workspace that qkv_paged_decode_attn_f4 takes. This
// entry point runs the same split pass and merge with the partials in a
// fixed array compiled into the library instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds QKV_STATIC_SCRATCH_BYTES of it until the process exits. In
// host code its name is only a host-side handle, not a device address, so
// the address is resolved with cudaGetSymbolAddress once per device (on the
// first call made with that device current) and cached.
#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_static_scratch[QKV_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices];  // device address of g_static_scratch, per device

// Device address of the array on the current device, or nullptr.
void* static_scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return nullptr;
    }
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int qkv_paged_decode_attn_f4_static(uint16_t* out, float* lse2_out, const uint16_t* q,
                                               const uint8_t* k_data, const uint16_t* k_scale,
                                               const uint8_t* v_data, const uint16_t* v_scale,
                                               const int32_t* page_table, const int32_t* seq_lens, int32_t n_seq,
                                               int32_t q_heads, int32_t kv_heads, int32_t head_dim,
                                               int32_t block_size, int32_t max_pages_per_seq, int64_t num_pages,
                                               float softmax_scale, int32_t num_splits, int32_t* device_status,
                                               qkv_stream_t stream) {
  if (n_seq < 0 || q_heads < 1 || kv_heads < 1 || head_dim < 1 || num_splits < 0) return QKV_EINVAL;
  if (n_seq == 0) return QKV_OK;
  const int32_t max_splits = num_splits > 0 ? num_splits : qkv_paged_decode_auto_splits(kv_heads, block_size);
  if (max_splits < 1) return QKV_EUNSUPPORTED;
  const size_t need = qkv_paged_decode_workspace_bytes(n_seq, q_heads, head_dim, max_splits);
  if (need == 0 || need > (size_t)QKV_STATIC_SCRATCH_BYTES) return QKV_EINVAL;  // partials do not fit
  void* scratch = static_scratch_address();
  if (!scratch) return QKV_ECUDA;
  // Nothing in the array has to start at zero: the split pass writes the
  // lse2 of every slot the merge reads, and the o row of every slot whose
  // lse2 is finite.
  return qkv_paged_decode_attn_f4(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens, n_seq,
                                  q_heads, kv_heads, head_dim, block_size, max_pages_per_seq, num_pages,
                                  softmax_scale, num_splits, max_splits, scratch, (size_t)QKV_STATIC_SCRATCH_BYTES,
                                  device_status, stream);
}
