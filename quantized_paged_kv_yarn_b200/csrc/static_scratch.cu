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
// the address is resolved with cudaGetSymbolAddress on the first call made
// with a device current, and cached for that device together with the
// identity of its CUDA context. A later call under another context of the
// device (after cudaDeviceReset, or once the primary context was released
// and created again, the module and its array are loaded anew) resolves the
// address again, and a failed launch drops the cached address.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace {

__device__ __align__(256) unsigned char g_static_scratch[QKV_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

struct Resolved {
  void* addr;               // device address of g_static_scratch
  unsigned long long ctx;   // unique id of the context it belongs to
};
std::mutex g_mu;
Resolved g_scratch[kMaxDevices];

using CtxGetCurrent = PFN_cuCtxGetCurrent_v4000;
using CtxGetId = PFN_cuCtxGetId_v12000;

// Unique id of the calling thread's current context (0 when it cannot be
// read: the cached address is then never trusted).
unsigned long long current_context_id() {
  static CtxGetCurrent get_current = nullptr;
  static CtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the array on the current device, or nullptr.
void* static_scratch_address(int& dev) {
  dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  // cudaGetSymbolAddress makes the device's primary context current if none
  // is; the context id is read after it
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long ctx = current_context_id();
  Resolved& r = g_scratch[dev];
  if (r.addr && ctx != 0 && r.ctx == ctx) return r.addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    r = Resolved{nullptr, 0};
    return nullptr;
  }
  ctx = current_context_id();
  r = Resolved{p, ctx};
  return p;
}

void forget_static_scratch(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return;
  std::lock_guard<std::mutex> lock(g_mu);
  g_scratch[dev] = Resolved{nullptr, 0};
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
  int dev = -1;
  void* scratch = static_scratch_address(dev);
  if (!scratch) return QKV_ECUDA;
  // Nothing in the array has to start at zero: the split pass writes the
  // lse2 of every slot the merge reads, and the o row of every slot whose
  // lse2 is finite.
  const int rc = qkv_paged_decode_attn_f4(out, lse2_out, q, k_data, k_scale, v_data, v_scale, page_table, seq_lens,
                                          n_seq, q_heads, kv_heads, head_dim, block_size, max_pages_per_seq,
                                          num_pages, softmax_scale, num_splits, max_splits, scratch,
                                          (size_t)QKV_STATIC_SCRATCH_BYTES, device_status, stream);
  if (rc == QKV_ECUDA) forget_static_scratch(dev);  // the next call resolves the address again
  return rc;
}
