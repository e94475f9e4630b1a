// decode_split_d128.cu -- the split-pass kernel instances for head_dim 128
// (device code in decode_split.cuh; the host side is in decode_split.cu).
#include "decode_split.cuh"

namespace qkv {
template const void* split_kernel<128>(int, int, bool, bool);
template size_t split_kernel_smem<128>(int);
}  // namespace qkv
