// Decode-attention variants for FP8 E4M3 caches (E4M3 -> f16 in registers,
// tensor-core tile math).  The FP8 tile math issues about twice the
// instructions per byte of the 16-bit path, so it runs more warps per SM to
// hide their latency, and 32-token tiles when blocks hold 32 tokens (one tile
// = one block) so the per-tile work (table lookup, softmax reductions,
// accumulator rescale) is spread over twice the bytes.
#include "attn_launch.cuh"

namespace pkv {
template <typename QT>
static pkv_status launch_fp8(const DecodeLaunchArgs& a, cudaStream_t s) {
    if (a.params->block_size % 32 == 0)
        return launch_decode<Cfg<uint8_t, QT, 128, Path::kFp8, 8, 2, 32>>(a, s);
    return launch_decode<Cfg<uint8_t, QT, 128, Path::kFp8, 12, 3>>(a, s);
}
pkv_status launch_decode_fp8_qf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_fp8<__half>(a, s);
}
pkv_status launch_decode_fp8_qbf16_d128(const DecodeLaunchArgs& a, cudaStream_t s) {
    return launch_fp8<__nv_bfloat16>(a, s);
}
}  // namespace pkv
