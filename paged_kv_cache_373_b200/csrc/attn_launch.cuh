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

// The decode grid with one of the two length-scan forms.
template <class C, bool kSuffix, bool kWideScan>
pkv_status launch_decode_grid(const DecodeLaunchArgs& a, const SuffixArg<kSuffix>& sx, cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};  // bit per device (< 64)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(pkv_decode_kernel<C, kSuffix, kWideScan>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   C::kSmemBytes);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "smem opt-in: %s", cudaGetErrorString(e));
        configured.fetch_or(bit);
    }
    const DecodeParams& p = *a.params;
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
        e = cudaLaunchKernelEx(&cfg, pkv_decode_kernel<C, kSuffix, kWideScan>, p, sx);
    } else {
        pkv_decode_kernel<C, kSuffix, kWideScan><<<a.grid, C::kWarps * 32, C::kSmemBytes, st>>>(p, sx);
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "decode launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

template <class C, bool kSuffix>
pkv_status launch_decode_k(const DecodeLaunchArgs& a, cudaStream_t st) {
    static_assert(C::kSmemBytes + sizeof(BlockScanSmem) <= 227 * 1024, "shared memory budget");
    const DecodeParams& p = *a.params;
    SuffixArg<kSuffix> sx{};
    if constexpr (kSuffix)
        sx = SuffixArg<true>{a.seq_start, a.part_o, a.part_ml, a.prefix_eff, a.cta_ticket, a.num_groups,
                             a.prefix_units, a.prefix_tile};
    // the length scans: each warp alone while one round of a warp's scan
    // covers the batch, else once per CTA
    const pkv_status ds = p.num_seqs > 32 * kScanPerLane ? launch_decode_grid<C, kSuffix, true>(a, sx, st)
                                                          : launch_decode_grid<C, kSuffix, false>(a, sx, st);
    if (ds != PKV_OK) return ds;
    if (kSuffix && a.skip_merge) return PKV_OK;  // the cascade's finish pass merges the split units
    cudaError_t e = cudaSuccess;
    // the merge kernel is a programmatic dependent launch: its CTAs start
    // while the decode grid drains, locate their unit from the lengths (which
    // the decode kernel does not write) and wait for the decode grid's results
    // only before reading the workspace
    const int64_t workers = (int64_t)a.grid * C::kWarps;
    cudaLaunchConfig_t cfg = {};
    // one CTA per worker boundary (a warp per head row), or for batches
    // whose length scan takes more than two rounds of a warp, 8 boundaries
    // per CTA located by one CTA-wide scan
    const bool wide = p.num_seqs > 2 * 32 * kScanPerLane;
    cfg.gridDim = dim3((unsigned)(wide ? (workers + kMergeWarps - 1) / kMergeWarps : workers));
    cfg.blockDim = dim3(32 * (wide ? kMergeWarps : p.hpu));
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (wide)
        e = cudaLaunchKernelEx(&cfg, pkv_merge_wide_kernel<typename C::q_t, C::D, C::kTT, kSuffix>, p, workers, sx);
    else
        e = cudaLaunchKernelEx(&cfg, pkv_merge_kernel<typename C::q_t, C::D, C::kTT, kSuffix>, p, workers, sx);
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
