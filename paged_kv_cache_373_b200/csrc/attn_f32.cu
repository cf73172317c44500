// Decode-attention variants for fp32 caches (CUDA-core consumer).
#include "attn_launch.cuh"

namespace pkv {
pkv_status launch_decode_f32_d64(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<float, float, 64, Path::kF32, 8, 2>>(a, s);
}
pkv_status launch_decode_f32_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<float, float, 128, Path::kF32, 4, 2>>(a, s);
}
}  // namespace pkv
