// attn_launch.cuh -- launcher template shared by the per-variant
// translation units (attn_*.cu): opt the kernel into its shared-memory size
// once per device, launch the decode kernel (one warp = one worker) and the
// split-merge kernel (one warp per worker boundary).
#pragma once

#include <atomic>
#include <cstdio>

#include "paged_attention.cuh"
#include "pkv_internal.h"

namespace pkv {

template <class C, bool kSuffix>
pkv_status launch_decode_k(const DecodeLaunchArgs& a, cudaStream_t st) {
    static_assert(C::kSmemBytes <= 227 * 1024, "shared memory budget");
    static std::atomic<unsigned long long> configured{0};  // bit per device (< 64)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(pkv_decode_kernel<C, kSuffix>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   C::kSmemBytes);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "smem opt-in: %s", cudaGetErrorString(e));
        configured.fetch_or(bit);
    }
    const DecodeParams& p = *a.params;
    SuffixArg<kSuffix> sx{};
    if constexpr (kSuffix) sx = SuffixArg<true>{a.seq_start, a.part_o, a.part_ml};
    cudaError_t e = cudaSuccess;
    if constexpr (kSuffix) {
        // the cascade suffix pass: a programmatic dependent of the prefix pass
        // (it may start on SMs the prefix pass leaves; see WaitPrimaryAtExit)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)a.grid);
        cfg.blockDim = dim3(C::kWarps * 32);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, pkv_decode_kernel<C, kSuffix>, p, sx);
    } else {
        pkv_decode_kernel<C, kSuffix><<<a.grid, C::kWarps * 32, C::kSmemBytes, st>>>(p, sx);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "decode launch: %s", cudaGetErrorString(e));
    // the merge kernel is a programmatic dependent launch: its CTAs start
    // while the decode grid drains, locate their unit from the lengths (which
    // the decode kernel does not write) and wait for the decode grid's results
    // only before reading the workspace
    const int64_t workers = (int64_t)a.grid * C::kWarps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)workers);
    cfg.blockDim = dim3(32 * p.hpu);  // a warp per head row
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, pkv_merge_kernel<typename C::q_t, C::D, C::kTT, kSuffix>, p,
                           workers, sx);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "merge launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

// Plain decode, or the cascade suffix pass when the call asks for it.
template <class C>
pkv_status launch_decode(const DecodeLaunchArgs& a, cudaStream_t st) {
    return a.suffix ? launch_decode_k<C, true>(a, st) : launch_decode_k<C, false>(a, st);
}

}  // namespace pkv
