// prefill.cu -- pkv_paged_prefill: chunked-prefill attention over the paged
// KV cache (ttlab.hopto.org "LLM KV cache 02", section 3: a long prompt is cut
// into chunks that share each step's token budget with decode tokens).  The
// chunk's K/V are already in the cache (pkv_reshape_and_cache); chunk token i
// of sequence s sits at position p = seq_lens[s] - C_s + i and attends to the
// cached tokens t <= p through the block table.
//
// Work unit: (sequence, kv head, 128 query rows); a row is a (chunk token,
// q head of the kv head's group) pair, so one K/V tile in shared memory serves
// all g heads of every token in the unit.  A CTA of 4 warps (thread = row):
//   - gathers the unit's 64-token K/V tiles through the table with 16-byte
//     cp.async (zero fill past the unit's last position, 2-stage ring) into
//     the 128-byte-swizzled layout the tensor core reads;
//   - one thread issues S = Q K^T on the 5th-generation tensor core
//     (tcgen05.mma, M = 128 rows, N = 64 tokens, accumulator in tensor
//     memory), every thread loads its row of S from tensor memory and runs
//     the online softmax in registers;
//   - P is written to shared memory (bf16: hi + lo parts, so P V keeps
//     fp32-level accuracy) and O_t = P V_t is issued (N = head_dim, V read
//     MN-major); each thread folds its row of O_t into its running output.
// Completion of each group of tensor-core products is signalled on an
// mbarrier (tcgen05.commit); every wait is bounded and a timeout sets
// PKV_DEVERR_TIMEOUT.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kPfRows = 128;   // query rows per unit (tensor-core M)
constexpr int kPfTok = 64;     // KV tokens per tile (N of S, K of P V)
constexpr int kPfStages = 2;   // K/V ring depth
constexpr int kPfThreads = 256;  // two threads per row: warps w and w + 4 share TMEM lanes

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

// Byte offset of 16-byte chunk c of row r in a [rows][cols] 16-bit tile kept
// as column blocks of 64 elements: block c / 8 holds rows x 128 bytes, and
// inside it 8-row groups of 1024 bytes with the 128-byte XOR swizzle.  This
// is the canonical swizzled layout of the tensor core's shared-memory
// operands (K-major rows for Q, K and P; MN-major for V).
__device__ __forceinline__ uint32_t tc_off(int r, int c, int rows) {
    return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor: start address, leading / stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16 with an fp32 accumulator.
template <bool kBf16>
__device__ __forceinline__ uint32_t tc_idesc(int M, int N, int b_mn_major) {
    const uint32_t fmt = kBf16 ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    const uint32_t z = 0;
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n"
                 ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(z));
}
__device__ __forceinline__ void tc_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for the mbarrier phase `parity`; false after 0.2 s of wall-clock time.
__device__ __forceinline__ bool tc_wait(uint32_t mbar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile("{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
                     "selp.b32 %0, 1, 0, P1;\n\t}\n"
                     : "=r"(ok) : "r"(mbar), "r"(parity) : "memory");
        if (ok) return true;
        if ((it & 63) == 63) {
            const uint64_t now = global_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > 200000000ull) return false;
        }
    }
}
// 16 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16-byte async copy; src_bytes = 0 writes zeros (no global read)
__device__ __forceinline__ void cp16_zfill(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void pf_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void pf_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename T, int D>
struct PfSmem {
    static constexpr int kQ = kPfRows * D * 2;
    static constexpr int kTile = kPfTok * D * 2;   // one K or V tile
    static constexpr int kP = kPfRows * kPfTok * 2;
    static constexpr int kParts = std::is_same<T, __nv_bfloat16>::value ? 2 : 1;  // P hi (+ lo)
    static constexpr int kBytes = kQ + 2 * kPfStages * kTile + kParts * kP + 1024;  // + alignment
    static constexpr int kTmemCols = 256;            // S (64 columns) + O_t (D columns)
};

template <typename T, int D>
__global__ void __launch_bounds__(kPfThreads, 1)
pkv_prefill_kernel(const PrefillParams p) {
    using SM = PfSmem<T, D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int CH = D / 8;  // 16-byte chunks per row
    extern __shared__ uint8_t pf_raw[];
    uint8_t* sm = pf_raw + ((1024 - (smem_u32(pf_raw) & 1023)) & 1023);  // 1024-byte aligned operands
    uint8_t* qsm = sm;
    uint8_t* ksm = qsm + SM::kQ;
    uint8_t* vsm = ksm + kPfStages * SM::kTile;
    uint8_t* psm = vsm + kPfStages * SM::kTile;  // P hi, then P lo (bf16)
    __shared__ __align__(8) uint64_t bars[2];     // S done, O_t done
    __shared__ uint32_t tmem_base;
    __shared__ float xmax[2][kPfRows];            // the two halves' row maxima (and, at the end, sums)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- the unit: kv head from the block index, then row tile u among all
    // sequences' row tiles (warp-parallel scan; every warp finds it)
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

    // ---- tensor memory and barriers
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(SM::kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // ---- q rows (zero past the chunk), with the first K/V tile
    for (int i = tid; i < kPfRows * CH; i += kPfThreads) {
        const int r = i / CH, c = i % CH;
        const int tl = r / p.g;
        const uint8_t* src = static_cast<const uint8_t*>(p.q);
        int nb = 0;
        if (tl < ntok) {
            src += ((int64_t)(q0 + tok0 + tl) * p.num_heads + (int64_t)kh * p.g + r % p.g) * (D * 2) + c * 16;
            nb = 16;
        }
        cp16_zfill(smem_u32(qsm + tc_off(r, c, kPfRows)), src, nb);
    }
    // each thread copies chunk cc of rows rr, rr + RSTEP, ... of a K/V tile;
    // the tile's physical blocks are read from the table one tile ahead of
    // their copies (the copies' asm is a compiler memory barrier)
    constexpr int RSTEP = kPfThreads / CH;
    constexpr int NIT = kPfTok / RSTEP;
    constexpr int NBLK = kPfTok / 16;
    const int rr = tid / CH, cc = tid % CH;
    const int lg_bs = p.bs == 16 ? 4 : 5;
    auto load_phys = [&](int kt, int (&ph)[NBLK]) {
#pragma unroll
        for (int jb = 0; jb < NBLK; ++jb) {
            const int t = kt * kPfTok + (jb << lg_bs);
            ph[jb] = (t < kv_end && (jb << lg_bs) < kPfTok) ? __ldg(trow + (t >> lg_bs)) : -1;
        }
    };
    auto issue_kv = [&](int kt, int stage, const int (&ph)[NBLK]) {
        uint8_t* kd = ksm + stage * SM::kTile;
        uint8_t* vd = vsm + stage * SM::kTile;
#pragma unroll
        for (int i = 0; i < NIT; ++i) {
            const int r = rr + RSTEP * i;
            const int t = kt * kPfTok + r;
            const int jb = r >> lg_bs;
            int phys = ph[0];
#pragma unroll
            for (int q = 1; q < NBLK; ++q) phys = jb == q ? ph[q] : phys;
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
            const uint32_t so = tc_off(r, cc, kPfTok);
            cp16_zfill(smem_u32(kd + so), ks, nb);
            cp16_zfill(smem_u32(vd + so), vs, nb);
        }
    };
    int phn[NBLK];
    load_phys(0, phn);
    issue_kv(0, 0, phn);
    pf_commit();
    if (nkv > 1) load_phys(1, phn);

    // ---- this thread's row and half: S columns [32 half, 32 half + 32), O
    // columns [half D / 2, (half + 1) D / 2)
    const int row = tid & (kPfRows - 1), half = tid >> 7;
    constexpr int SH = kPfTok / 2, DH = D / 2;
    const int pos = (row / p.g < ntok) ? ctx + tok0 + row / p.g : -1;
    float o[DH];
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] = 0.f;
    float m = -INFINITY, l = 0.f;

    __syncthreads();  // barriers initialised, tensor memory allocated
    tc_after_sync();
    const uint32_t tmem = tmem_base;
    const uint32_t tS = tmem, tO = tmem + kPfTok;                  // columns
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;  // this warp's 32 lanes
    const uint32_t id_s = tc_idesc<kBf16>(kPfRows, kPfTok, 0);
    const uint32_t id_o = tc_idesc<kBf16>(kPfRows, D, 1);
    bool timed_out = false;

#pragma unroll 1
    for (int kt = 0; kt < nkv; ++kt) {
        pf_wait<0>();
        fence_async_smem();  // the copies, visible to the tensor core
        __syncthreads();     // tile kt (and q) complete; every thread done with tile kt - 1
        tc_after_sync();
        const int st = kt % kPfStages;
        if (tid == 0) {  // S = Q K^T
            const uint32_t qa = smem_u32(qsm), kb = smem_u32(ksm + st * SM::kTile);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                tc_mma(tS, tc_desc(qa + (kk >> 2) * kPfRows * 128 + (kk & 3) * 32, 16, 1024),
                       tc_desc(kb + (kk >> 2) * kPfTok * 128 + (kk & 3) * 32, 16, 1024), id_s, kk > 0);
            tc_commit(smem_u32(&bars[0]));
        }
        if (kt + 1 < nkv) {  // the next tile into the other stage (its last reader, tile kt - 1, is done)
            issue_kv(kt + 1, (kt + 1) % kPfStages, phn);
            if (kt + 2 < nkv) load_phys(kt + 2, phn);
        }
        pf_commit();
        timed_out |= !tc_wait(smem_u32(&bars[0]), kt & 1);
        tc_after_sync();
        // ---- this row's scores: scale (log2 domain), causal mask, online
        // softmax; the row maximum is combined with the other half's
        float sc[SH];
#pragma unroll
        for (int c0 = 0; c0 < SH; c0 += 16) tc_ld16(tS + lane_addr + half * SH + c0, sc + c0);
        const int t0 = kt * kPfTok + half * SH;
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < SH; ++c) {
            sc[c] = t0 + c <= pos ? sc[c] * p.scale_log2 : -INFINITY;
            mx4[c & 3] = fmaxf(mx4[c & 3], sc[c]);
        }
        xmax[half][row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        __syncthreads();
        const float mx = fmaxf(xmax[0][row], xmax[1][row]);
        const float mn = fmaxf(m, mx);
        const float ref = mn == -INFINITY ? 0.f : mn;  // a row with nothing attended yet
        const float alpha = ex2(m - ref);
        m = mn;
        float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < SH; ++c) {
            sc[c] = ex2(sc[c] - ref);
            ls4[c & 3] += sc[c];
        }
        l = l * alpha + ((ls4[0] + ls4[1]) + (ls4[2] + ls4[3]));  // this half's share of the sum
        // ---- this half of P to shared memory (K-major rows; bf16 as hi + lo parts)
#pragma unroll
        for (int c8 = 0; c8 < SH / 8; ++c8) {
            uint32_t h[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a = sc[c8 * 8 + 2 * e], b = sc[c8 * 8 + 2 * e + 1];
                h[e] = pack2<kBf16>(a, b);
                if constexpr (kBf16) {
                    const float2 hf = unpack2<true>(h[e]);
                    lo[e] = pack2<true>(a - hf.x, b - hf.y);
                }
            }
            const uint32_t off = tc_off(row, half * (SH / 8) + c8, kPfRows);
            *reinterpret_cast<uint4*>(psm + off) = make_uint4(h[0], h[1], h[2], h[3]);
            if constexpr (kBf16) *reinterpret_cast<uint4*>(psm + SM::kP + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();  // P complete; every thread has read its row of S
        tc_after_sync();
        if (tid == 0) {  // O_t = P V (hi, then lo)
            const uint32_t vb = smem_u32(vsm + st * SM::kTile);
#pragma unroll
            for (int part = 0; part < SM::kParts; ++part) {
                const uint32_t pa = smem_u32(psm + part * SM::kP);
#pragma unroll
                for (int kk = 0; kk < kPfTok / 16; ++kk)
                    tc_mma(tO, tc_desc(pa + kk * 32, 16, 1024), tc_desc(vb + kk * 2048, kPfTok * 128, 1024), id_o,
                           (part > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(smem_u32(&bars[1]));
        }
        timed_out |= !tc_wait(smem_u32(&bars[1]), kt & 1);
        tc_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 16) {
            float ov[16];
            tc_ld16(tO + lane_addr + half * DH + c0, ov);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[c0 + e] = o[c0 + e] * alpha + ov[e];
        }
        tc_before_sync();
        if (__syncthreads_or(timed_out)) {
            timed_out = true;
            break;
        }
    }
    pf_wait<0>();

    // ---- normalise (the two halves' sums combined) and store this half of the row
    xmax[half][row] = l;
    __syncthreads();
    const float lt = xmax[0][row] + xmax[1][row];
    if (timed_out) {
        if (tid == 0) raise_error(p.err, PKV_DEVERR_TIMEOUT);
    } else if (pos >= 0) {
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        T* out = static_cast<T*>(p.out) +
                 ((int64_t)(q0 + tok0 + row / p.g) * p.num_heads + (int64_t)kh * p.g + row % p.g) * D + half * DH;
#pragma unroll
        for (int c8 = 0; c8 < DH / 8; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = pack2<kBf16>(o[c8 * 8 + 2 * e] * inv, o[c8 * 8 + 2 * e + 1] * inv);
            *reinterpret_cast<uint4*>(out + c8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    tc_before_sync();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(SM::kTmemCols));
}

template <typename T, int D>
pkv_status launch_prefill(const PrefillParams& p, int64_t grid, cudaStream_t st) {
    constexpr int kSmem = PfSmem<T, D>::kBytes;
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
    pkv_prefill_kernel<T, D><<<(unsigned)grid, kPfThreads, kSmem, st>>>(p);
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
