// Decode-attention variants for FP8 E4M3 caches (E4M3 -> f16 in registers,
// tensor-core consumer).
#include "attn_launch.cuh"

namespace pkv {
pkv_status launch_decode_fp8_qf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<uint8_t, __half, 128, Path::kFp8, 8, 4>>(a, s);
}
pkv_status launch_decode_fp8_qbf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<uint8_t, __nv_bfloat16, 128, Path::kFp8, 8, 4>>(a, s);
}
}  // namespace pkv
