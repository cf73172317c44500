// Decode-attention variants for FP8 E4M3 caches (E4M3 -> f16 in registers,
// tensor-core tile math).  The FP8 tile math issues about twice the
// instructions per byte of the 16-bit path, so it runs 12 warps per SM
// (3-stage rings) to hide their latency: 14 % faster than 8 warps on a B200.
#include "attn_launch.cuh"

namespace pkv {
pkv_status launch_decode_fp8_qf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<uint8_t, __half, 128, Path::kFp8, 12, 3>>(a, s);
}
pkv_status launch_decode_fp8_qbf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_decode<Cfg<uint8_t, __nv_bfloat16, 128, Path::kFp8, 12, 3>>(a, s);
}
}  // namespace pkv
