// Decode-attention variants for f16 caches (tensor-core consumer).
#include "attn_launch.cuh"

namespace pkv {
pkv_status launch_decode_f16_d64(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<__half, __half, 64, Path::kMma16, kWarps16, 4>>(a, s);
}
pkv_status launch_decode_f16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<__half, __half, 128, Path::kMma16, kWarps16, 2>>(a, s);
}
}  // namespace pkv
