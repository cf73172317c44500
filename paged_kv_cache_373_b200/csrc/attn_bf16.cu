// Decode-attention variants for bf16 caches (tensor-core consumer).
#include "attn_launch.cuh"

namespace pkv {
pkv_status launch_decode_bf16_d64(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<__nv_bfloat16, __nv_bfloat16, 64, Path::kMma16, kWarps16, 4>>(a, s);
}
pkv_status launch_decode_bf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<__nv_bfloat16, __nv_bfloat16, 128, Path::kMma16, kWarps16, 2>>(a, s);
}
}  // namespace pkv
