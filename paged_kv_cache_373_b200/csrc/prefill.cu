// prefill.cu -- pkv_paged_prefill: chunked-prefill attention over the paged
// KV cache (ttlab.hopto.org "LLM KV cache 02", section 3: a long prompt is cut
// into chunks that share each step's token budget with decode tokens).  The
// chunk's K/V are already in the cache (pkv_reshape_and_cache); chunk token i
// of sequence s sits at position p = seq_lens[s] - C_s + i and attends to the
// cached tokens t <= p through the block table.
//
// Work unit: (sequence, kv head, tile of 64 query rows); a row is a (chunk
// token, q head of the kv head's group) pair, so one K/V tile in shared
// memory serves all g heads of every token in the unit.  A CTA of 4 warps
// streams the unit's K/V tiles of 64 tokens (paged gather with 16-byte
// cp.async, zero fill past the valid range, a 3-stage ring, XOR-swizzled
// rows) and each warp runs the online softmax for its 16 rows with
// mma.sync m16n8k16: S = Q K^T (q rows as A, K rows as B via ldmatrix),
// O += P V (P re-packed from the S accumulators, V via ldmatrix.trans).  For
// bf16, P is carried as hi + lo bf16 parts so P V keeps fp32-level accuracy.
// Tiles past a warp's last position are skipped (causal).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kPfWarps = 4;
constexpr int kPfRows = 16 * kPfWarps;  // query rows per unit
constexpr int kPfTok = 64;              // KV tokens per tile
constexpr int kPfStages = 3;            // K/V ring depth

struct PrefillParams {
    void* out;
    const void* q;
    const uint8_t* kc;
    const uint8_t* vc;
    const int32_t* tables;
    const int32_t* seq_lens;
    const int32_t* qstart;
    int* err;
    int64_t num_blocks;
    int num_seqs, num_heads, num_kv_heads, g, mbps, bs;
    float scale_log2;
};

// byte offset of 16-byte chunk c of row r in a [rows][D] 16-bit tile; the
// chunk index is XOR-swizzled with the row inside each 128-byte group so the
// eight row addresses of an ldmatrix hit eight different bank groups
template <int D>
__device__ __forceinline__ uint32_t pf_off(int r, int c) {
    return (uint32_t)(r * (D * 2) + (((c & ~7) | ((c ^ r) & 7)) << 4));
}

// 16-byte async copy; src_bytes = 0 writes zeros (no global read)
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void pf_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void pf_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// bf16 pair of (a, b) - hi, where hi is their bf16 rounding
__device__ __forceinline__ uint32_t lo_part(float a, float b, uint32_t hi) {
    const float2 h = unpack2<true>(hi);
    return pack2<true>(a - h.x, b - h.y);
}

template <typename T, int D>
__global__ void __launch_bounds__(kPfWarps * 32, 2)
pkv_prefill_kernel(const PrefillParams p) {
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int CH = D / 8;            // 16-byte chunks per row
    constexpr int KS = D / 16;           // k-steps of q.k
    constexpr int NT = kPfTok / 8;       // n-tiles of S
    constexpr int DT = D / 8;            // n-tiles of O
    constexpr int TILE = kPfTok * D * 2; // bytes of one K or V tile
    extern __shared__ __align__(128) uint8_t pf_smem[];
    uint8_t* qsm = pf_smem;                       // kPfRows x D
    uint8_t* ksm = pf_smem + kPfRows * D * 2;     // kPfStages stages
    uint8_t* vsm = ksm + kPfStages * TILE;        // kPfStages stages
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    // ---- the unit: kv head from the block index, then the row tile u among
    // all sequences' row tiles (warp-parallel scan; every warp finds it)
    const int kh = (int)(blockIdx.x % p.num_kv_heads);
    const int64_t u = blockIdx.x / p.num_kv_heads;
    int s = -1, j = 0;
    {
        int64_t base = 0;
        for (int s0 = 0; s0 < p.num_seqs && s < 0; s0 += 32) {
            const int si = s0 + lane;
            int nrt = 0;
            if (si < p.num_seqs) {
                const int C = __ldg(p.qstart + si + 1) - __ldg(p.qstart + si);
                if (C < 0 && blockIdx.x == 0 && warp == 0) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
                nrt = C > 0 ? (int)(((int64_t)C * p.g + kPfRows - 1) / kPfRows) : 0;
            }
            int incl = nrt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            const int64_t lo = base + incl - nrt;
            const unsigned hit = __ballot_sync(kFull, nrt > 0 && u >= lo && u < lo + nrt);
            if (hit) {
                const int src = __ffs(hit) - 1;
                s = s0 + src;
                const int64_t l0 = __shfl_sync(kFull, lo, src);
                const int nr = __shfl_sync(kFull, nrt, src);
                j = nr - 1 - (int)(u - l0);  // a sequence's last (heaviest) row tile first
            }
            base += __shfl_sync(kFull, incl, 31);
        }
    }
    if (s < 0) return;  // past the last unit

    const int q0 = __ldg(p.qstart + s);
    const int C = __ldg(p.qstart + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (L < C || L > p.mbps * p.bs) {
        if (tid == 0) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
        return;
    }
    const int ctx = L - C;
    const int tpu = kPfRows / p.g;           // chunk tokens per unit (g divides 16)
    const int tok0 = j * tpu;
    const int ntok = min(tpu, C - tok0);
    const int kv_end = ctx + tok0 + ntok;    // the unit reads KV tokens [0, kv_end)
    const int nkv = (kv_end + kPfTok - 1) / kPfTok;
    const int32_t* trow = p.tables + (int64_t)s * p.mbps;

    // ---- q rows (zero past the chunk), with the first K/V tile
    for (int i = tid; i < kPfRows * CH; i += kPfWarps * 32) {
        const int r = i / CH, c = i % CH;
        const int tl = r / p.g;
        const uint8_t* src = static_cast<const uint8_t*>(p.q);
        int nb = 0;
        if (tl < ntok) {
            src += ((int64_t)(q0 + tok0 + tl) * p.num_heads + (int64_t)kh * p.g + r % p.g) * (D * 2) + c * 16;
            nb = 16;
        }
        cp16_zfill(smem_u32(qsm + pf_off<D>(r, c)), src, nb);
    }
    // each thread copies chunk cc of rows rr, rr + RSTEP, ... of a K/V tile.
    // The tile's (at most 4) physical blocks are read from the table one tile
    // ahead of their copies: the copies' asm is a compiler memory barrier,
    // so table reads interleaved with them would each stall in turn.
    constexpr int RSTEP = kPfWarps * 32 / CH;
    constexpr int NIT = kPfTok / RSTEP;
    constexpr int NBLK = kPfTok / 16;         // blocks per tile at block_size 16
    const int rr = tid / CH, cc = tid % CH;
    const int lg_bs = p.bs == 16 ? 4 : 5;
    auto load_phys = [&](int kt, int (&ph)[NBLK]) {
#pragma unroll
        for (int j = 0; j < NBLK; ++j) {
            const int t = kt * kPfTok + (j << lg_bs);
            ph[j] = (t < kv_end && (j << lg_bs) < kPfTok) ? __ldg(trow + (t >> lg_bs)) : -1;
        }
    };
    auto issue_kv = [&](int kt, int stage, const int (&ph)[NBLK]) {
        uint8_t* kd = ksm + stage * TILE;
        uint8_t* vd = vsm + stage * TILE;
#pragma unroll
        for (int i = 0; i < NIT; ++i) {
            const int r = rr + RSTEP * i;
            const int t = kt * kPfTok + r;
            const int j = r >> lg_bs;
            const int phys = j == 0 ? ph[0] : j == 1 ? ph[1] : j == 2 ? ph[2] : ph[3];
            const uint8_t* ks = p.kc;
            const uint8_t* vs = p.vc;
            int nb = 0;
            if (t < kv_end) {
                if (phys >= 0 && phys < p.num_blocks) {
                    const int64_t off =
                        (((int64_t)phys * p.bs + (t & (p.bs - 1))) * p.num_kv_heads + kh) * (D * 2) + cc * 16;
                    ks += off;
                    vs += off;
                    nb = 16;
                } else if (cc == 0) {
                    raise_error(p.err, PKV_DEVERR_BLOCK_ID);
                }
            }
            const uint32_t so = pf_off<D>(r, cc);
            cp16_zfill(smem_u32(kd + so), ks, nb);
            cp16_zfill(smem_u32(vd + so), vs, nb);
        }
    };
    // async groups: {q, tile 0}, {tile 1}, then one group per iteration
    // (possibly empty), so "all but the newest group done" means tile kt landed
    int phn[NBLK];
    load_phys(0, phn);
    issue_kv(0, 0, phn);
    pf_commit();
    if (nkv > 1) {
        load_phys(1, phn);
        issue_kv(1, 1, phn);
    }
    pf_commit();
    if (nkv > 2) load_phys(2, phn);

    // ---- this thread's two rows (gid, gid + 8 of the warp's 16)
    const int r0 = warp * 16 + gid, r1 = r0 + 8;
    const int pos0 = (r0 / p.g < ntok) ? ctx + tok0 + r0 / p.g : -1;
    const int pos1 = (r1 / p.g < ntok) ? ctx + tok0 + r1 / p.g : -1;
    const int wlast = min(ntok - 1, (warp * 16 + 15) / p.g);
    const int wmax = ((warp * 16) / p.g < ntok) ? ctx + tok0 + wlast : -1;  // last position of the warp

    uint32_t qa[KS][4];
    float o[DT][4];
#pragma unroll
    for (int d = 0; d < DT; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

#pragma unroll 1
    for (int kt = 0; kt < nkv; ++kt) {
        pf_wait<1>();
        __syncthreads();  // tile kt visible to all warps; all are done with tile kt - 1
        if (kt + 2 < nkv) issue_kv(kt + 2, (kt + 2) % kPfStages, phn);  // refills tile kt - 1's stage
        pf_commit();
        if (kt + 3 < nkv) load_phys(kt + 3, phn);  // in flight during this tile's math
        if (kt == 0) {
#pragma unroll
            for (int kk = 0; kk < KS; ++kk)
                ldsm_x4(qa[kk], smem_u32(qsm + pf_off<D>(warp * 16 + (lane & 15), 2 * kk + (lane >> 4))));
        }
        const int t0 = kt * kPfTok;
        if (t0 <= wmax) {
            const uint8_t* kt_s = ksm + (kt % kPfStages) * TILE;
            const uint8_t* vt_s = vsm + (kt % kPfStages) * TILE;
            float sc[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
            // k-steps outer: the NT accumulators are independent chains
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
                for (int np = 0; np < NT / 2; ++np) {
                    uint32_t b[4];
                    const int tr = np * 16 + (lane & 7) + ((lane >> 4) << 3);
                    ldsm_x4(b, smem_u32(kt_s + pf_off<D>(tr, 2 * kk + ((lane >> 3) & 1))));
                    mma16816<kBf16>(sc[2 * np], qa[kk], b[0], b[1]);
                    mma16816<kBf16>(sc[2 * np + 1], qa[kk], b[2], b[3]);
                }
            }
            // scale (log2 domain), causal mask, row maxima
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int t = t0 + n * 8 + 2 * tig;
                sc[n][0] = t <= pos0 ? sc[n][0] * p.scale_log2 : -INFINITY;
                sc[n][1] = t + 1 <= pos0 ? sc[n][1] * p.scale_log2 : -INFINITY;
                sc[n][2] = t <= pos1 ? sc[n][2] * p.scale_log2 : -INFINITY;
                sc[n][3] = t + 1 <= pos1 ? sc[n][3] * p.scale_log2 : -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(sc[n][0], sc[n][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[n][2], sc[n][3]));
            }
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
            }
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float ref0 = mn0 == -INFINITY ? 0.f : mn0;  // rows with nothing attended yet
            const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
            const float a0 = ex2(m0 - ref0), a1 = ex2(m1 - ref1);
            m0 = mn0;
            m1 = mn1;
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                sc[n][0] = ex2(sc[n][0] - ref0);
                sc[n][1] = ex2(sc[n][1] - ref0);
                sc[n][2] = ex2(sc[n][2] - ref1);
                sc[n][3] = ex2(sc[n][3] - ref1);
                ls0 += sc[n][0] + sc[n][1];
                ls1 += sc[n][2] + sc[n][3];
            }
            l0 = l0 * a0 + ls0;
            l1 = l1 * a1 + ls1;
#pragma unroll
            for (int d = 0; d < DT; ++d) {
                o[d][0] *= a0; o[d][1] *= a0;
                o[d][2] *= a1; o[d][3] *= a1;
            }
            // O += P V, 16 tokens per k-step
#pragma unroll
            for (int kk = 0; kk < NT / 2; ++kk) {
                uint32_t pa[4], pl[4];
                pa[0] = pack2<kBf16>(sc[2 * kk][0], sc[2 * kk][1]);
                pa[1] = pack2<kBf16>(sc[2 * kk][2], sc[2 * kk][3]);
                pa[2] = pack2<kBf16>(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                pa[3] = pack2<kBf16>(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
                if constexpr (kBf16) {  // the residuals P - bf16(P)
                    pl[0] = lo_part(sc[2 * kk][0], sc[2 * kk][1], pa[0]);
                    pl[1] = lo_part(sc[2 * kk][2], sc[2 * kk][3], pa[1]);
                    pl[2] = lo_part(sc[2 * kk + 1][0], sc[2 * kk + 1][1], pa[2]);
                    pl[3] = lo_part(sc[2 * kk + 1][2], sc[2 * kk + 1][3], pa[3]);
                }
                // each V fragment is loaded once; the lo products of the
                // previous fragment pair follow the hi products of the next
                uint32_t bp[4];
#pragma unroll
                for (int dp = 0; dp < DT / 2; ++dp) {
                    uint32_t b[4];
                    const int tr = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                    ldsm_x4_trans(b, smem_u32(vt_s + pf_off<D>(tr, 2 * dp + (lane >> 4))));
                    mma16816<kBf16>(o[2 * dp], pa, b[0], b[1]);
                    mma16816<kBf16>(o[2 * dp + 1], pa, b[2], b[3]);
                    if constexpr (kBf16) {
                        if (dp > 0) {
                            mma16816<kBf16>(o[2 * dp - 2], pl, bp[0], bp[1]);
                            mma16816<kBf16>(o[2 * dp - 1], pl, bp[2], bp[3]);
                        }
                        bp[0] = b[0]; bp[1] = b[1]; bp[2] = b[2]; bp[3] = b[3];
                    }
                }
                if constexpr (kBf16) {
                    mma16816<kBf16>(o[DT - 2], pl, bp[0], bp[1]);
                    mma16816<kBf16>(o[DT - 1], pl, bp[2], bp[3]);
                }
            }
        }
    }
    pf_wait<0>();

    // ---- normalise and store the valid rows
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, off);
        l1 += __shfl_xor_sync(kFull, l1, off);
    }
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    T* out = static_cast<T*>(p.out);
    if (pos0 >= 0) {
        T* row = out + ((int64_t)(q0 + tok0 + r0 / p.g) * p.num_heads + (int64_t)kh * p.g + r0 % p.g) * D;
#pragma unroll
        for (int d = 0; d < DT; ++d)
            *reinterpret_cast<uint32_t*>(row + d * 8 + 2 * tig) = pack2<kBf16>(o[d][0] * i0, o[d][1] * i0);
    }
    if (pos1 >= 0) {
        T* row = out + ((int64_t)(q0 + tok0 + r1 / p.g) * p.num_heads + (int64_t)kh * p.g + r1 % p.g) * D;
#pragma unroll
        for (int d = 0; d < DT; ++d)
            *reinterpret_cast<uint32_t*>(row + d * 8 + 2 * tig) = pack2<kBf16>(o[d][2] * i1, o[d][3] * i1);
    }
}

template <typename T, int D>
pkv_status launch_prefill(const PrefillParams& p, int64_t grid, cudaStream_t st) {
    constexpr int kSmem = kPfRows * D * 2 + 2 * kPfStages * kPfTok * D * 2;
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(PKV_ECUDA, "cudaGetDevice");
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(pkv_prefill_kernel<T, D>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "prefill smem opt-in: %s", cudaGetErrorString(e));
        configured.fetch_or(bit);
    }
    pkv_prefill_kernel<T, D><<<(unsigned)grid, kPfWarps * 32, kSmem, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "prefill launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_paged_prefill(void* out, const void* query, pkv_dtype q_dtype,
                                        const void* key_cache, const void* value_cache,
                                        pkv_dtype cache_dtype, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* seq_lens,
                                        const int32_t* query_start, int num_seqs,
                                        int64_t num_query_tokens, int num_heads, int num_kv_heads,
                                        int head_dim, int block_size, int64_t num_blocks, float scale,
                                        pkv_stream_t stream) {
    if (num_seqs < 0 || num_query_tokens < 0) return fail(PKV_EINVAL, "negative size");
    if (num_kv_heads <= 0 || num_heads <= 0 || num_heads % num_kv_heads)
        return fail(PKV_EINVAL, "num_heads must be a positive multiple of num_kv_heads");
    const int g = num_heads / num_kv_heads;
    if (16 % g) return fail(PKV_EUNSUPPORTED, "heads per kv head %d (1, 2, 4, 8 or 16)", g);
    if (head_dim != 64 && head_dim != 128) return fail(PKV_EUNSUPPORTED, "head_dim %d", head_dim);
    if (block_size != 16 && block_size != 32) return fail(PKV_EUNSUPPORTED, "block_size %d", block_size);
    if (!(cache_dtype == PKV_F16 || cache_dtype == PKV_BF16) || q_dtype != cache_dtype)
        return fail(PKV_EUNSUPPORTED, "prefill needs f16 or bf16 caches and q of the same dtype");
    if (num_blocks <= 0 || max_blocks_per_seq <= 0) return fail(PKV_EINVAL, "empty pool or table");
    if (!(scale > 0.f) || !(scale < INFINITY)) return fail(PKV_EINVAL, "scale must be positive and finite");
    if (num_seqs == 0 || num_query_tokens == 0) return PKV_OK;
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !query_start)
        return fail(PKV_EINVAL, "null pointer");
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PKV_EINVAL, "buffers must be 16-byte aligned");
    int* err = device_error_word();
    if (!err) return fail(PKV_ECUDA, "device error word unavailable");
    PrefillParams p{};
    p.out = out;
    p.q = query;
    p.kc = static_cast<const uint8_t*>(key_cache);
    p.vc = static_cast<const uint8_t*>(value_cache);
    p.tables = block_tables;
    p.seq_lens = seq_lens;
    p.qstart = query_start;
    p.err = err;
    p.num_blocks = num_blocks;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.g = g;
    p.mbps = max_blocks_per_seq;
    p.bs = block_size;
    p.scale_log2 = scale * 1.4426950408889634f;
    // row tiles: sum_s ceil(C_s g / 64) <= ceil(T g / 64) + S
    const int64_t units = (num_query_tokens * g + kPfRows - 1) / kPfRows + num_seqs;
    const int64_t grid = units * num_kv_heads;
    if (grid > 0x7fffffffLL) return fail(PKV_EUNSUPPORTED, "too many query rows");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cache_dtype == PKV_F16)
        return head_dim == 64 ? launch_prefill<__half, 64>(p, grid, cs) : launch_prefill<__half, 128>(p, grid, cs);
    return head_dim == 64 ? launch_prefill<__nv_bfloat16, 64>(p, grid, cs)
                          : launch_prefill<__nv_bfloat16, 128>(p, grid, cs);
}
