// pkv_internal.h -- host-side declarations shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/pkv.h"

namespace pkv {

// Device address of the static error word on the current device (null on failure).
int* device_error_word();

// Record a message for pkv_last_error_message() and return `st`.
pkv_status fail(pkv_status st, const char* fmt, ...);

int dtype_bytes(pkv_dtype d);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DecodeParams;  // paged_attention.cuh

struct DecodeLaunchArgs {
    const DecodeParams* params;
    int grid;  // CTAs of the persistent grid
};

// One launcher per kernel variant (attn_*.cu).
pkv_status launch_decode_f32_d64(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_f32_d128(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_f16_d64(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_f16_d128(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_bf16_d64(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_bf16_d128(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_fp8_qf16_d128(const DecodeLaunchArgs&, cudaStream_t);
pkv_status launch_decode_fp8_qbf16_d128(const DecodeLaunchArgs&, cudaStream_t);

}  // namespace pkv
