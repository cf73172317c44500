// cache_ops.cu -- pkv_reshape_and_cache and pkv_copy_blocks.
//
// reshape_and_cache: zwxr.cn section 3.1 (a token occupies a slot once it is
// produced) and 3.2 (slot = physical block * block_size + offset).  One
// thread moves one 16-byte chunk of a token's K row and the same chunk of its
// V row; rows are contiguous in both layouts ([T, Hkv, D] and
// [NB, bs, Hkv, D]), so slot -> row address is slot * Hkv * D.
//
// copy_blocks: zwxr.cn section 3.4 copy-on-write.  One CTA copies one whole
// block of one layer's K or V cache with 16-byte vector loads/stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {

__global__ void reshape_copy_kernel(const uint8_t* __restrict__ key, const uint8_t* __restrict__ value,
                                    uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                    const int64_t* __restrict__ slots, int64_t num_tokens,
                                    int64_t num_slots, int row_bytes, int* err) {
    const int cpr = row_bytes / 16;
    const int64_t total = num_tokens * cpr;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / cpr;
        const int c = (int)(idx % cpr);
        const int64_t slot = __ldg(slots + i);
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (c == 0) raise_error(err, PKV_DEVERR_SLOT);
            continue;
        }
        const uint4 k = __ldg(reinterpret_cast<const uint4*>(key + i * row_bytes) + c);
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(value + i * row_bytes) + c);
        reinterpret_cast<uint4*>(kc + slot * row_bytes)[c] = k;
        reinterpret_cast<uint4*>(vc + slot * row_bytes)[c] = v;
    }
}

template <typename SrcT>
__device__ __forceinline__ float to_f32(SrcT x) { return static_cast<float>(x); }

// 16 source elements -> 16 E4M3 codes: RNE + saturation of the IEEE fp32
// quotient x / scale.
template <typename SrcT>
__device__ __forceinline__ uint4 quant16(const SrcT* src, float scale) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = __fdiv_rn(to_f32(src[4 * j + 0]), scale);
        const float b = __fdiv_rn(to_f32(src[4 * j + 1]), scale);
        const float c = __fdiv_rn(to_f32(src[4 * j + 2]), scale);
        const float d = __fdiv_rn(to_f32(src[4 * j + 3]), scale);
        w[j] = (uint32_t)f32x2_to_e4m3x2(a, b) | ((uint32_t)f32x2_to_e4m3x2(c, d) << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <typename SrcT>
__global__ void reshape_fp8_kernel(const SrcT* __restrict__ key, const SrcT* __restrict__ value,
                                   uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                   const int64_t* __restrict__ slots, int64_t num_tokens,
                                   int64_t num_slots, int row_elems, const float* k_scale,
                                   const float* v_scale, int* err) {
    const int cpr = row_elems / 16;  // 16 elements -> one 16-byte chunk of codes
    const int64_t total = num_tokens * cpr;
    const float ks = __ldg(k_scale), vs = __ldg(v_scale);
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = idx / cpr;
        const int c = (int)(idx % cpr);
        const int64_t slot = __ldg(slots + i);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (c == 0) raise_error(err, PKV_DEVERR_SLOT);
            continue;
        }
        alignas(16) SrcT kb[16], vb[16];
        constexpr int kVec = 16 * (int)sizeof(SrcT) / 16;
#pragma unroll
        for (int j = 0; j < kVec; ++j) {
            reinterpret_cast<uint4*>(kb)[j] =
                __ldg(reinterpret_cast<const uint4*>(key + i * row_elems + 16 * c) + j);
            reinterpret_cast<uint4*>(vb)[j] =
                __ldg(reinterpret_cast<const uint4*>(value + i * row_elems + 16 * c) + j);
        }
        reinterpret_cast<uint4*>(kc + slot * row_elems)[c] = quant16(kb, ks);
        reinterpret_cast<uint4*>(vc + slot * row_elems)[c] = quant16(vb, vs);
    }
}

constexpr int kMaxLayers = 128;
struct LayerPtrs {
    uint8_t* k[kMaxLayers];
    uint8_t* v[kMaxLayers];
};

__global__ void __launch_bounds__(256)
copy_blocks_kernel(const LayerPtrs ptrs, const int64_t* __restrict__ mapping, int64_t num_blocks,
                   int64_t block_bytes, int* err) {
    const int64_t pair = blockIdx.x;
    const int layer = blockIdx.y >> 1;
    const int which = blockIdx.y & 1;
    const int64_t src = __ldg(mapping + 2 * pair), dst = __ldg(mapping + 2 * pair + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0) raise_error(err, PKV_DEVERR_COPY_ID);
        return;
    }
    uint8_t* base = which ? ptrs.v[layer] : ptrs.k[layer];
    const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
    uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
    const int64_t n = block_bytes / 16;
    int64_t i = threadIdx.x;
    for (; i + 3 * blockDim.x < n; i += 4 * blockDim.x) {  // 4 loads in flight per thread
        const uint4 a = __ldg(s + i), b = __ldg(s + i + blockDim.x);
        const uint4 c = __ldg(s + i + 2 * blockDim.x), e = __ldg(s + i + 3 * blockDim.x);
        d[i] = a; d[i + blockDim.x] = b; d[i + 2 * blockDim.x] = c; d[i + 3 * blockDim.x] = e;
    }
    for (; i < n; i += blockDim.x) d[i] = __ldg(s + i);
}

static int grid_for(int64_t work, int threads) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 16;
    return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_reshape_and_cache(const void* key, const void* value, pkv_dtype src_dtype,
                                            void* key_cache, void* value_cache, pkv_dtype cache_dtype,
                                            const int64_t* slot_mapping, int64_t num_tokens,
                                            int64_t num_blocks, int block_size, int num_kv_heads,
                                            int head_dim, const float* k_scale, const float* v_scale,
                                            pkv_stream_t stream) {
    if (num_tokens < 0) return fail(PKV_EINVAL, "num_tokens < 0");
    if (num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0)
        return fail(PKV_EINVAL, "num_blocks, block_size and num_kv_heads must be positive");
    if (head_dim != 64 && head_dim != 128) return fail(PKV_EUNSUPPORTED, "head_dim %d", head_dim);
    if (dtype_bytes(src_dtype) == 0 || dtype_bytes(cache_dtype) == 0)
        return fail(PKV_EINVAL, "unknown dtype");
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (!fp8 && src_dtype != cache_dtype)
        return fail(PKV_EUNSUPPORTED, "non-FP8 caches need src_dtype == cache_dtype");
    if (fp8 && src_dtype == PKV_FP8_E4M3) return fail(PKV_EUNSUPPORTED, "FP8 source");
    if (num_tokens == 0) return PKV_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping)
        return fail(PKV_EINVAL, "null pointer");
    if (fp8 && (!k_scale || !v_scale)) return fail(PKV_EINVAL, "FP8 cache needs k_scale and v_scale");
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PKV_EINVAL, "buffers must be 16-byte aligned");
    int* err = device_error_word();
    if (!err) return fail(PKV_ECUDA, "device error word unavailable");
    const int row_elems = num_kv_heads * head_dim;
    const int64_t num_slots = num_blocks * block_size;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int threads = 256;
    if (!fp8) {
        const int row_bytes = row_elems * dtype_bytes(src_dtype);
        const int grid = grid_for(num_tokens * (row_bytes / 16), threads);
        reshape_copy_kernel<<<grid, threads, 0, st>>>(
            static_cast<const uint8_t*>(key), static_cast<const uint8_t*>(value),
            static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), slot_mapping,
            num_tokens, num_slots, row_bytes, err);
    } else {
        const int grid = grid_for(num_tokens * (row_elems / 16), threads);
        switch (src_dtype) {
        case PKV_F32:
            reshape_fp8_kernel<float><<<grid, threads, 0, st>>>(
                static_cast<const float*>(key), static_cast<const float*>(value),
                static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), slot_mapping,
                num_tokens, num_slots, row_elems, k_scale, v_scale, err);
            break;
        case PKV_F16:
            reshape_fp8_kernel<__half><<<grid, threads, 0, st>>>(
                static_cast<const __half*>(key), static_cast<const __half*>(value),
                static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), slot_mapping,
                num_tokens, num_slots, row_elems, k_scale, v_scale, err);
            break;
        default:
            reshape_fp8_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
                static_cast<const __nv_bfloat16*>(key), static_cast<const __nv_bfloat16*>(value),
                static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache), slot_mapping,
                num_tokens, num_slots, row_elems, k_scale, v_scale, err);
            break;
        }
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "reshape_and_cache launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

extern "C" pkv_status pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                                      const int64_t* block_mapping, int64_t num_pairs, int64_t num_blocks,
                                      size_t block_bytes, pkv_stream_t stream) {
    if (num_pairs < 0) return fail(PKV_EINVAL, "num_pairs < 0");
    if (num_layers < 1 || num_layers > kMaxLayers)
        return fail(PKV_EINVAL, "num_layers must be in [1, %d]", kMaxLayers);
    if (num_blocks <= 0) return fail(PKV_EINVAL, "num_blocks must be positive");
    if (block_bytes == 0 || block_bytes % 16 != 0)
        return fail(PKV_EINVAL, "block_bytes must be a positive multiple of 16");
    if (num_pairs == 0) return PKV_OK;
    if (num_pairs > 0x7fffffffLL) return fail(PKV_EUNSUPPORTED, "too many pairs");
    if (!key_caches || !value_caches || !block_mapping) return fail(PKV_EINVAL, "null pointer");
    LayerPtrs ptrs{};
    for (int l = 0; l < num_layers; ++l) {
        if (!key_caches[l] || !value_caches[l]) return fail(PKV_EINVAL, "null cache pointer (layer %d)", l);
        if (!aligned16(key_caches[l]) || !aligned16(value_caches[l]))
            return fail(PKV_EINVAL, "caches must be 16-byte aligned");
        ptrs.k[l] = static_cast<uint8_t*>(key_caches[l]);
        ptrs.v[l] = static_cast<uint8_t*>(value_caches[l]);
    }
    int* err = device_error_word();
    if (!err) return fail(PKV_ECUDA, "device error word unavailable");
    const dim3 grid((unsigned)num_pairs, 2u * (unsigned)num_layers);
    copy_blocks_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        ptrs, block_mapping, num_blocks, (int64_t)block_bytes, err);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "copy_blocks launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}
