// swap.cu -- pkv_swap_blocks: whole-block copies between two block pools that
// may live in different memory spaces (device HBM, or page-locked host memory
// reached by the GPU through unified addressing).  This is the data movement
// of preemption by swapping (zwxr.cn section 4.3): the KV blocks of a
// preempted sequence move to host memory, and move back, to any free blocks,
// once device blocks are free again.
//
// One launch covers every (pair, layer, K/V): the kernel reads and writes
// the pools directly, so a swap of many small blocks costs one launch rather
// than one DMA call per block; each thread keeps four 16-byte loads in flight
// to cover the latency of the host link.
#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kMaxSwapLayers = 128;
struct SwapPtrs {
    const uint8_t* src_k[kMaxSwapLayers];
    const uint8_t* src_v[kMaxSwapLayers];
    uint8_t* dst_k[kMaxSwapLayers];
    uint8_t* dst_v[kMaxSwapLayers];
};

// grid: (pairs, 2 * layers); CTA (p, 2l + w) copies block mapping[p][0] of
// layer l's K (w = 0) or V (w = 1) pool into block mapping[p][1].
__global__ void __launch_bounds__(256)
swap_blocks_kernel(const SwapPtrs ptrs, const int64_t* __restrict__ mapping,
                   int64_t src_blocks, int64_t dst_blocks, int64_t block_bytes, int* err) {
    const int64_t pair = blockIdx.x;
    const int layer = blockIdx.y >> 1;
    const int which = blockIdx.y & 1;
    const int64_t src = mapping[2 * pair], dst = mapping[2 * pair + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (threadIdx.x == 0) raise_error(err, PKV_DEVERR_COPY_ID);
        return;
    }
    const uint8_t* sb = which ? ptrs.src_v[layer] : ptrs.src_k[layer];
    uint8_t* db = which ? ptrs.dst_v[layer] : ptrs.dst_k[layer];
    const uint4* s = reinterpret_cast<const uint4*>(sb + src * block_bytes);
    uint4* d = reinterpret_cast<uint4*>(db + dst * block_bytes);
    const int64_t n = block_bytes / 16;
    int64_t i = threadIdx.x;
    for (; i + 3 * blockDim.x < n; i += 4 * blockDim.x) {
        const uint4 a = s[i], b = s[i + blockDim.x], c = s[i + 2 * blockDim.x], e = s[i + 3 * blockDim.x];
        d[i] = a; d[i + blockDim.x] = b; d[i + 2 * blockDim.x] = c; d[i + 3 * blockDim.x] = e;
    }
    for (; i < n; i += blockDim.x) d[i] = s[i];
}

// The pool pointer must be device memory of the current device or
// page-locked host memory mapped into the device's address space.
pkv_status check_reachable(const void* ptr, int dev, const char* what, int layer) {
    cudaPointerAttributes a;
    const cudaError_t e = cudaPointerGetAttributes(&a, ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PKV_EINVAL, "%s (layer %d): not a CUDA-visible pointer", what, layer);
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
        if (a.device != dev)
            return fail(PKV_EUNSUPPORTED, "%s (layer %d): memory of device %d, launching on %d", what,
                        layer, a.device, dev);
        return PKV_OK;
    }
    if (a.type == cudaMemoryTypeHost) {
        if (a.devicePointer != ptr)
            return fail(PKV_EUNSUPPORTED, "%s (layer %d): host memory not mapped at the same address", what,
                        layer);
        return PKV_OK;
    }
    return fail(PKV_EINVAL, "%s (layer %d): pageable host memory (pin it first)", what, layer);
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                                      int64_t dst_num_blocks, const void* const* src_key_caches,
                                      const void* const* src_value_caches, int64_t src_num_blocks,
                                      int num_layers, const int64_t* block_mapping, int64_t num_pairs,
                                      size_t block_bytes, pkv_stream_t stream) {
    if (num_pairs < 0) return fail(PKV_EINVAL, "num_pairs < 0");
    if (num_layers < 1 || num_layers > kMaxSwapLayers)
        return fail(PKV_EINVAL, "num_layers must be in [1, %d]", kMaxSwapLayers);
    if (src_num_blocks <= 0 || dst_num_blocks <= 0) return fail(PKV_EINVAL, "num_blocks must be positive");
    if (block_bytes == 0 || block_bytes % 16 != 0)
        return fail(PKV_EINVAL, "block_bytes must be a positive multiple of 16");
    if (num_pairs == 0) return PKV_OK;
    if (num_pairs > 0x7fffffffLL) return fail(PKV_EUNSUPPORTED, "too many pairs");
    if (!dst_key_caches || !dst_value_caches || !src_key_caches || !src_value_caches || !block_mapping)
        return fail(PKV_EINVAL, "null pointer");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    if (pkv_status st = check_reachable(block_mapping, dev, "block_mapping", 0)) return st;
    SwapPtrs ptrs{};  // 4 KB of kernel parameters at 128 layers
    for (int l = 0; l < num_layers; ++l) {
        const void* q[4] = {dst_key_caches[l], dst_value_caches[l], src_key_caches[l], src_value_caches[l]};
        static const char* names[4] = {"dst key cache", "dst value cache", "src key cache", "src value cache"};
        for (int j = 0; j < 4; ++j) {
            if (!q[j]) return fail(PKV_EINVAL, "null %s (layer %d)", names[j], l);
            if (!aligned16(q[j])) return fail(PKV_EINVAL, "%s (layer %d) must be 16-byte aligned", names[j], l);
            if (pkv_status st = check_reachable(q[j], dev, names[j], l)) return st;
        }
        ptrs.dst_k[l] = static_cast<uint8_t*>(dst_key_caches[l]);
        ptrs.dst_v[l] = static_cast<uint8_t*>(dst_value_caches[l]);
        ptrs.src_k[l] = static_cast<const uint8_t*>(src_key_caches[l]);
        ptrs.src_v[l] = static_cast<const uint8_t*>(src_value_caches[l]);
    }
    int* err = device_error_word();
    if (!err) return fail(PKV_ECUDA, "device error word unavailable");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)num_pairs, 2u * (unsigned)num_layers);
    swap_blocks_kernel<<<grid, 256, 0, cs>>>(ptrs, block_mapping, src_num_blocks, dst_num_blocks,
                                             (int64_t)block_bytes, err);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "swap launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}
