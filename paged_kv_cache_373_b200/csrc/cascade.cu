// cascade.cu -- host side of pkv_paged_attention_decode_cascade: workspace
// layout, validation, and the launch sequence of the passes in cascade.cuh.
#include <algorithm>
#include <atomic>

#include "cascade.cuh"
#include "cascade_tc.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kMaxSmem = 227 * 1024;

// Launch `kern` as a programmatic dependent of the previous kernel on `st`
// (the kernel waits for it with griddepcontrol.wait before reading its results).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct CascadeLayout {
    int g, rows, nt, row_chunks;
    size_t dec, pre_seg_o, pre_seg_ml, seq_start, member_info, prefix_eff, suf_o, suf_ml, pre_o, pre_ml,
        seq_grp, total;
};

bool cascade_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int num_groups,
                    int max_group_size, int num_ctas, CascadeLayout* L) {
    if (num_groups < 0 || max_group_size < 1 || num_kv_heads <= 0 || num_heads % num_kv_heads) return false;
    const size_t dec = decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, num_ctas);
    if (dec == 0) return false;
    int grid = num_ctas;
    if (grid == 0 && (cudaGetDevice(&grid) != cudaSuccess ||
                      cudaDeviceGetAttribute(&grid, cudaDevAttrMultiProcessorCount, grid) != cudaSuccess))
        return false;
    L->g = num_heads / num_kv_heads;
    L->rows = max_group_size * L->g;
    L->nt = L->rows > 8 ? 4 : 2;
    const int rpu = 8 * L->nt;
    L->row_chunks = (L->rows + rpu - 1) / rpu;
    const size_t units = (size_t)num_groups * num_kv_heads * L->row_chunks;
    const size_t segs = (size_t)grid * kMaxWarpsPerCta + units;
    size_t off = align256(dec);
    L->dec = dec;
    L->pre_seg_o = off;  off = align256(off + segs * rpu * head_dim * sizeof(float));
    L->pre_seg_ml = off; off = align256(off + segs * rpu * sizeof(float2));
    L->seq_start = off;  off = align256(off + (size_t)(num_seqs + 1) * sizeof(int32_t));  // + the suffix CTA ticket
    L->member_info = off; off = align256(off + (size_t)num_seqs * sizeof(int4));
    L->prefix_eff = off; off = align256(off + (size_t)num_groups * sizeof(int32_t));
    L->suf_o = off;      off = align256(off + (size_t)num_seqs * num_heads * head_dim * sizeof(float));
    L->suf_ml = off;     off = align256(off + (size_t)num_seqs * num_heads * sizeof(float2));
    const size_t prows = (size_t)num_groups * num_kv_heads * L->rows;
    L->pre_o = off;      off = align256(off + prows * head_dim * sizeof(float));
    L->pre_ml = off;     off = align256(off + prows * sizeof(float2));
    L->seq_grp = off;    off = align256(off + (size_t)num_seqs * sizeof(int2));
    L->total = off;
    return true;
}

template <class C, int NT>
pkv_status launch_prefix(const DecodeParams& p, const CascadeParams& c, int grid, cudaStream_t st) {
    constexpr int kSmem = C::kWarps * (C::kStages * C::kStageBytes + 2 * 8 * NT * C::kRowBytes) + 1024;
    static_assert(kSmem <= kMaxSmem, "prefix kernel shared memory");
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(pkv_prefix_kernel<C, NT>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "prefix smem opt-in: %s", cudaGetErrorString(e));
        configured.fetch_or(bit);
    }
    const cudaError_t e = launch_dependent(pkv_prefix_kernel<C, NT>, dim3(grid), dim3(C::kWarps * 32), kSmem, st, p, c);
    if (e != cudaSuccess) return fail(PKV_ECUDA, "prefix launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

// warps per CTA of the prefix pass (2-stage K/V rings + 2 query slots): 8
// for two row tiles; 7 for four (their query slots are twice as large).
// Measured on cfg5: more warps beat deeper rings (6 warps x 2 stages 68.7 us,
// 5 x 3 81.6 us).
constexpr int prefix_warps(int nt) { return nt == 2 ? 8 : 7; }
constexpr int kPrefixStages = 2;

template <typename T, int D>
pkv_status launch_prefix_t(const DecodeParams& p, const CascadeParams& c, int nt, int grid, cudaStream_t st) {
    if (nt == 2) return launch_prefix<Cfg<T, T, D, Path::kMma16, prefix_warps(2), kPrefixStages>, 2>(p, c, grid, st);
    return launch_prefix<Cfg<T, T, D, Path::kMma16, prefix_warps(4), kPrefixStages>, 4>(p, c, grid, st);
}

// The prefix pass on the tensor core (head_dim 128, 32-row units, 16-bit
// caches, power-of-two blocks of 16 to 64 tokens).
template <typename T>
pkv_status launch_prefix_tc(const DecodeParams& p, const CascadeParams& c, int grid, cudaStream_t st) {
    static_assert(kTcSmem <= kMaxSmem, "tensor-core prefix pass shared memory");
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(pkv_prefix_tc_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kTcSmem);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "prefix smem opt-in: %s", cudaGetErrorString(e));
        configured.fetch_or(bit);
    }
    const cudaError_t e = launch_dependent(pkv_prefix_tc_kernel<T>, dim3(grid), dim3(kTcThreads), kTcSmem, st, p, c);
    if (e != cudaSuccess) return fail(PKV_ECUDA, "prefix launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

template <typename QT, int D>
pkv_status launch_combine(const DecodeParams& p, const CascadeParams& c, int nt, cudaStream_t st) {
    const dim3 grid((unsigned)p.num_seqs, (unsigned)((p.num_heads + 7) / 8));  // a warp per (member, head)
    const cudaError_t e = nt == 2 ? launch_dependent(pkv_cascade_combine_kernel<QT, D, 2>, grid, dim3(256), 0, st, p, c)
                                  : launch_dependent(pkv_cascade_combine_kernel<QT, D, 4>, grid, dim3(256), 0, st, p, c);
    if (e != cudaSuccess) return fail(PKV_ECUDA, "combine launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

template <typename QT, int D>
pkv_status launch_finish(const DecodeParams& p, const CascadeParams& c, int nt, cudaStream_t st) {
    const dim3 grid((unsigned)p.num_seqs, (unsigned)((p.num_heads + 7) / 8));  // a warp per (sequence, head)
    const cudaError_t e = nt == 2 ? launch_dependent(pkv_cascade_finish_kernel<QT, D, 2>, grid, dim3(256), 0, st, p, c)
                                  : launch_dependent(pkv_cascade_finish_kernel<QT, D, 4>, grid, dim3(256), 0, st, p, c);
    if (e != cudaSuccess) return fail(PKV_ECUDA, "finish launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" size_t pkv_paged_attention_cascade_workspace_bytes(int num_seqs, int num_heads,
                                                              int num_kv_heads, int head_dim,
                                                              int num_groups, int max_group_size,
                                                              int num_ctas) {
    CascadeLayout L;
    if (!cascade_layout(num_seqs, num_heads, num_kv_heads, head_dim, num_groups, max_group_size,
                        num_ctas, &L))
        return 0;
    return L.total;
}

extern "C" pkv_status pkv_paged_attention_decode_cascade(
    void* out, const void* query, pkv_dtype q_dtype, const void* key_cache, const void* value_cache,
    pkv_dtype cache_dtype, const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
    int num_seqs, const int32_t* group_offsets, const int32_t* group_members,
    const int32_t* group_prefix_lens, int num_groups, int max_group_size, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
    const float* k_scale, const float* v_scale, void* workspace, size_t workspace_bytes, int num_ctas,
    pkv_stream_t stream) {
    if (num_groups < 0 || max_group_size < 1) return fail(PKV_EINVAL, "num_groups < 0 or max_group_size < 1");
    if (num_groups > 0 && (!group_offsets || !group_members || !group_prefix_lens))
        return fail(PKV_EINVAL, "null group array");
    const bool rows_path = (cache_dtype == PKV_F16 || cache_dtype == PKV_BF16) && q_dtype == cache_dtype;
    CascadeLayout L;
    if (num_seqs > 0 && !cascade_layout(num_seqs, num_heads, num_kv_heads, head_dim, num_groups,
                                        max_group_size, num_ctas, &L))
        return fail(PKV_EINVAL, "invalid shapes");
    if (num_seqs > 0 && workspace_bytes < L.total)
        return fail(PKV_EINVAL, "cascade workspace too small: %zu < %zu bytes", workspace_bytes, L.total);
    // the suffix pass is the ordinary decode path on the first workspace region
    DecodeParams p;
    DecodeLauncher launch;
    int grid = 0;
    pkv_status st = decode_prepare(&p, &launch, &grid, out, query, q_dtype, key_cache, value_cache,
                                   cache_dtype, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                   num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                                   k_scale, v_scale, workspace, num_seqs > 0 ? L.dec : 0, num_ctas);
    if (st != PKV_OK || num_seqs == 0) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    DecodeLaunchArgs a{&p, grid};
    if (num_groups == 0 || !rows_path) return launch(a, cs);  // no sharing to exploit: plain decode

    uint8_t* base = static_cast<uint8_t*>(workspace);
    CascadeParams c{};
    c.grp_offsets = group_offsets;
    c.grp_members = group_members;
    c.grp_prefix = group_prefix_lens;
    c.prefix_eff = reinterpret_cast<int32_t*>(base + L.prefix_eff);
    c.seq_start = reinterpret_cast<int32_t*>(base + L.seq_start);
    c.member_info = reinterpret_cast<int4*>(base + L.member_info);
    c.pre_o = reinterpret_cast<float*>(base + L.pre_o);
    c.pre_ml = reinterpret_cast<float2*>(base + L.pre_ml);
    c.suf_o = reinterpret_cast<float*>(base + L.suf_o);
    c.suf_ml = reinterpret_cast<float2*>(base + L.suf_ml);
    c.num_groups = num_groups;
    c.rows = L.rows;
    c.row_chunks = L.row_chunks;
    c.pre_seg_o = reinterpret_cast<const float*>(base + L.pre_seg_o);
    c.pre_seg_ml = reinterpret_cast<const float2*>(base + L.pre_seg_ml);
    c.seq_grp = reinterpret_cast<int2*>(base + L.seq_grp);
    c.suffix_workers = (int64_t)grid * kWarps16;
    // the prefix pass on the tensor core where its shape allows, else on mma.sync
    const bool tc_prefix = head_dim == kTcD && L.nt == 4 && block_size >= 16 && block_size <= kTcTok / 2 &&
                           (block_size & (block_size - 1)) == 0;
    c.prefix_workers = tc_prefix ? (int64_t)grid : (int64_t)grid * prefix_warps(L.nt);
    c.prefix_tile = tc_prefix ? kTcTok : 16;
    // The tensor-core prefix pass (one CTA per SM) and the suffix pass of a
    // finish-pass batch run side by side on disjoint SMs, in proportion to
    // their tokens; otherwise the suffix pass takes the SMs as the prefix
    // pass frees them.
    c.split_grid = tc_prefix && num_seqs <= 32 * kScanPerLane && grid >= 8 ? grid : 0;

    // seq_start and, after it, the suffix pass's CTA ticket
    pkv_cascade_zero_kernel<<<(unsigned)std::min(148, (num_seqs + 256) / 256), 256, 0, cs>>>(c.seq_start, num_seqs + 1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "zero launch: %s", cudaGetErrorString(e));
    e = launch_dependent(pkv_cascade_setup_kernel, dim3(num_groups), dim3(256), 0, cs, p, c);
    if (e != cudaSuccess) return fail(PKV_ECUDA, "setup launch: %s", cudaGetErrorString(e));

    DecodeParams pp = p;  // prefix pass: its own split segments
    pp.ws_o = reinterpret_cast<float*>(base + L.pre_seg_o);
    pp.ws_ml = reinterpret_cast<float2*>(base + L.pre_seg_ml);
    if (tc_prefix)
        st = cache_dtype == PKV_F16 ? launch_prefix_tc<__half>(pp, c, grid, cs)
                                    : launch_prefix_tc<__nv_bfloat16>(pp, c, grid, cs);
    else if (cache_dtype == PKV_F16)
        st = head_dim == 64 ? launch_prefix_t<__half, 64>(pp, c, L.nt, grid, cs)
                            : launch_prefix_t<__half, 128>(pp, c, L.nt, grid, cs);
    else
        st = head_dim == 64 ? launch_prefix_t<__nv_bfloat16, 64>(pp, c, L.nt, grid, cs)
                            : launch_prefix_t<__nv_bfloat16, 128>(pp, c, L.nt, grid, cs);
    if (st != PKV_OK) return st;

    // suffix pass: members from their shared-prefix end, partial outputs.
    // Batches whose length scan takes one round of a warp end with the
    // finish pass, which merges the suffix pass's split units itself (no
    // merge kernel between them); larger ones with the merge and combine
    // passes.
    const bool direct = num_seqs <= 32 * kScanPerLane;
    DecodeLaunchArgs sa{&p, grid, true, c.seq_start, c.suf_o, c.suf_ml, direct};
    if (c.split_grid > 0) {
        sa.prefix_eff = c.prefix_eff;
        sa.cta_ticket = c.seq_start + num_seqs;
        sa.num_groups = num_groups;
        sa.prefix_units = num_kv_heads * L.row_chunks;
        sa.prefix_tile = kTcTok;
    }
    if ((st = launch(sa, cs)) != PKV_OK) return st;

    if (direct) {
        if (cache_dtype == PKV_F16)
            return head_dim == 64 ? launch_finish<__half, 64>(p, c, L.nt, cs)
                                  : launch_finish<__half, 128>(p, c, L.nt, cs);
        return head_dim == 64 ? launch_finish<__nv_bfloat16, 64>(p, c, L.nt, cs)
                              : launch_finish<__nv_bfloat16, 128>(p, c, L.nt, cs);
    }
    if (cache_dtype == PKV_F16)
        return head_dim == 64 ? launch_combine<__half, 64>(p, c, L.nt, cs)
                              : launch_combine<__half, 128>(p, c, L.nt, cs);
    return head_dim == 64 ? launch_combine<__nv_bfloat16, 64>(p, c, L.nt, cs)
                          : launch_combine<__nv_bfloat16, 128>(p, c, L.nt, cs);
}
