// pkv_internal.h -- host-side declarations shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>
#include <vector>

#include "../../include/pkv.h"

namespace pkv {

// Device address of a file-scope __device__ symbol in the current context,
// cached per context (keyed by cuCtxGetId): the first call in a context does
// the cudaGetSymbolAddress lookup; null on failure.
struct SymbolCache {
    std::mutex mu;
    std::vector<std::pair<unsigned long long, void*>> entries;
};
void* symbol_address(const void* symbol, SymbolCache* cache);

// Device address of the static error word in the current context (null on failure).
int* device_error_word();

// Record a message for pkv_last_error_message() and return `st`.
pkv_status fail(pkv_status st, const char* fmt, ...);

int dtype_bytes(pkv_dtype d);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DecodeParams;  // paged_attention.cuh

struct DecodeLaunchArgs {
    const DecodeParams* params;
    int grid;            // CTAs of the persistent grid
    bool suffix = false; // cascade suffix pass: the fields below are used
    const int32_t* seq_start = nullptr;  // first attended token per sequence
    float* part_o = nullptr;             // partial outputs of sequences with a start > 0
    float2* part_ml = nullptr;
    bool skip_merge = false;             // suffix pass: split units left to the cascade's finish pass
    // suffix pass beside the prefix pass (prefix_tile > 0; see SuffixArg)
    const int32_t* prefix_eff = nullptr;
    int* cta_ticket = nullptr;
    int num_groups = 0, prefix_units = 0, prefix_tile = 0;
};

using DecodeLauncher = pkv_status (*)(const DecodeLaunchArgs&, cudaStream_t);

// Validate the arguments of pkv_paged_attention_decode and fill the kernel
// parameters, the variant's launcher and the grid size (pkv_api.cu).
pkv_status decode_prepare(DecodeParams* p, DecodeLauncher* launch, int* grid, void* out,
                          const void* query, pkv_dtype q_dtype, const void* key_cache,
                          const void* value_cache, pkv_dtype cache_dtype, const int32_t* block_tables,
                          int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                          const float* k_scale, const float* v_scale, void* workspace,
                          size_t workspace_bytes, int num_ctas);
size_t decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int num_ctas);

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
