// rope.cu -- YaRN rotary table and partial NEOX rotary (sm_100a).
//
// Sources: mistral.rs PR "YaRN rope scaling, 4-bit F4 packed KV cache, and
// hybrid paged attention for Qwen3.5-Next long-context serving", section 1
// (YaRN for a partial rotary resolved as llama.cpp does: corr_dims ramp from
// beta_fast / beta_slow, net table scale 1 + 0.1 ln(factor)); ignis docs
// "context-and-speculation", --model-rope-scaling (auto factor rule; the
// attention factor on queries and keys alike).
#include <math.h>

#include "common.cuh"

namespace qkv {

constexpr int MAX_ROT_HALF = 256;

struct YarnDev {
  double base, factor, orig, beta_fast, beta_slow, ext, attn;
  int rot;
};

// Angle step of pair j and the table scale, in double.
__device__ double yarn_theta(const YarnDev& p, int j, double* mscale) {
  const int d = p.rot;
  const double s = p.factor;
  const double ext = p.ext < 0 ? (s > 1.0 ? 1.0 : 0.0) : p.ext;
  *mscale = p.attn > 0 ? p.attn : (s > 1.0 ? 1.0 + 0.1 * log(s) : 1.0);
  // pair index where a frequency completes `beta` turns over the trained context
  const double two_pi = 6.283185307179586476925286766559;
  const double c_fast = d * log(p.orig / (p.beta_fast * two_pi)) / (2.0 * log(p.base));
  const double c_slow = d * log(p.orig / (p.beta_slow * two_pi)) / (2.0 * log(p.base));
  const double low = fmax(0.0, floor(c_fast));
  const double high = fmin((double)(d - 1), ceil(c_slow));
  const double omega = pow(p.base, -2.0 * j / d);
  const double y = fmin(1.0, fmax(0.0, (j - low) / fmax(0.001, high - low)));
  const double ramp = (1.0 - y) * ext;
  return (omega / s) * (1.0 - ramp) + omega * ramp;
}

// One block of 256 threads per 256 consecutive table entries (row-major
// [n_pos][rot/2]); the angle steps are computed once per block.
__global__ void __launch_bounds__(256) yarn_table_kernel(YarnDev p, int64_t pos_start, int64_t n_pos,
                                                         float* __restrict__ cos_out,
                                                         float* __restrict__ sin_out) {
  pdl_wait();  // the decode step reads the table before it waits: no early start of the successor
  __shared__ double s_theta[MAX_ROT_HALF];
  __shared__ double s_ms;
  const int half = p.rot / 2;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    double ms;
    s_theta[j] = yarn_theta(p, j, &ms);
    if (j == 0) s_ms = ms;
  }
  __syncthreads();
  const int64_t total = n_pos * half;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int64_t row = i / half;
  const int j = (int)(i - row * half);
  const double a = (double)(pos_start + row) * s_theta[j];
  double sn, cs;
  sincos(a, &sn, &cs);
  cos_out[i] = (float)(s_ms * cs);
  sin_out[i] = (float)(s_ms * sn);
}

// One warp per (token, head). Lanes walk the rotated pairs, then copy the
// pass-through dims when the output is a different buffer.
__global__ void __launch_bounds__(256) rope_apply_kernel(const __nv_bfloat16* x_in,  // may alias x_out
                                                         __nv_bfloat16* x_out,
                                                         const int64_t* __restrict__ positions, int n_tok,
                                                         int n_heads, int head_dim, int rot,
                                                         const float* __restrict__ cos_tab,
                                                         const float* __restrict__ sin_tab,
                                                         int64_t tab_start, int64_t tab_len,
                                                         int32_t* status) {
  pdl_release();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (item >= (int64_t)n_tok * n_heads) return;
  const int64_t tok = item / n_heads;
  const __nv_bfloat16* xi = x_in + item * head_dim;
  __nv_bfloat16* xo = x_out + item * head_dim;
  const int half = rot / 2;
  const int64_t row = positions[tok] - tab_start;
  const bool ok = row >= 0 && row < tab_len;
  if (!ok && lane == 0) flag(status, QKV_DEV_BAD_POSITION);
  for (int j = lane; j < half; j += 32) {
    const float x0 = __bfloat162float(xi[j]), x1 = __bfloat162float(xi[j + half]);
    if (ok) {
      const float c = cos_tab[row * half + j], s = sin_tab[row * half + j];
      xo[j] = __float2bfloat16_rn(rot_first(x0, x1, c, s));
      xo[j + half] = __float2bfloat16_rn(rot_second(x0, x1, c, s));
    } else {
      xo[j] = xi[j];
      xo[j + half] = xi[j + half];
    }
  }
  if (xi != xo)
    for (int j = rot + lane; j < head_dim; j += 32) xo[j] = xi[j];
}

}  // namespace qkv

using namespace qkv;

extern "C" double qkv_yarn_auto_factor(int64_t max_context, int64_t orig_max_pos) {
  if (max_context <= 0 || orig_max_pos <= 0) return -1.0;
  if (max_context <= orig_max_pos) return 0.0;
  const double f = (double)max_context / (double)orig_max_pos;
  return f > 64.0 ? -1.0 : f;
}

extern "C" int qkv_yarn_rope_table(const qkv_yarn_params* params, int64_t pos_start, int64_t n_pos,
                                   float* cos_out, float* sin_out, qkv_stream_t stream) {
  if (!params || !cos_out || !sin_out || n_pos < 0 || pos_start < 0) return QKV_EINVAL;
  const qkv_yarn_params& q = *params;
  if (q.rot_dim < 2 || (q.rot_dim & 1) || q.rot_dim / 2 > MAX_ROT_HALF) return QKV_EINVAL;
  if (!(q.factor >= 1.0) || !(q.rope_base > 1.0) || q.orig_max_pos <= 0) return QKV_EINVAL;
  if (!(q.beta_fast > 0) || !(q.beta_slow > 0)) return QKV_EINVAL;
  if (n_pos == 0) return QKV_OK;
  YarnDev p{q.rope_base, q.factor, (double)q.orig_max_pos, q.beta_fast, q.beta_slow,
            q.ext_factor, q.attn_factor, q.rot_dim};
  const int64_t total = n_pos * (q.rot_dim / 2);
  const int64_t blocks = (total + 255) / 256;
  if (blocks > 0x7fffffff) return QKV_EINVAL;
  void* args[] = {&p, &pos_start, &n_pos, &cos_out, &sin_out};
  if (launch_pdl((const void*)yarn_table_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}

extern "C" int qkv_rope_apply(const uint16_t* x_in, uint16_t* x_out, const int64_t* positions, int32_t n_tok,
                              int32_t n_heads, int32_t head_dim, int32_t rot_dim, const float* cos_tab,
                              const float* sin_tab, int64_t table_pos_start, int64_t table_len,
                              int32_t* device_status, qkv_stream_t stream) {
  if (n_tok == 0 || n_heads == 0) return QKV_OK;  // nothing to do; pointers may be NULL
  if (!x_in || !x_out || !positions || !cos_tab || !sin_tab) return QKV_EINVAL;
  if (n_tok < 0 || n_heads < 0 || head_dim < 2 || (head_dim & 1) || rot_dim < 2 || (rot_dim & 1) ||
      rot_dim > head_dim || table_len < 0)
    return QKV_EINVAL;
  if (x_in != x_out) {
    const size_t bytes = (size_t)n_tok * n_heads * head_dim * 2;
    const char *a = (const char*)x_in, *b = (const char*)x_out;
    if (a < b + bytes && b < a + bytes) return QKV_EINVAL;
  }
  const int64_t items = (int64_t)n_tok * n_heads;
  if (items == 0) return QKV_OK;
  const int64_t blocks = (items + 7) / 8;
  const __nv_bfloat16* xi = reinterpret_cast<const __nv_bfloat16*>(x_in);
  __nv_bfloat16* xo = reinterpret_cast<__nv_bfloat16*>(x_out);
  int nt = n_tok, nh = n_heads, hd = head_dim, rd = rot_dim;
  void* args[] = {&xi, &xo, &positions, &nt, &nh, &hd, &rd, &cos_tab, &sin_tab, &table_pos_start, &table_len,
                  &device_status};
  if (launch_pdl((const void*)rope_apply_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, args) != cudaSuccess) {
    (void)cudaGetLastError();
    return QKV_ECUDA;
  }
  return QKV_OK;
}
