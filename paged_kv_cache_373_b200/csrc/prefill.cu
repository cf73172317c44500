// prefill.cu -- pkv_paged_prefill: chunked-prefill attention over the paged
// KV cache (ttlab.hopto.org "LLM KV cache 02", section 3: a long prompt is cut
// into chunks that share each step's token budget with decode tokens).  The
// chunk's K/V are already in the cache (pkv_reshape_and_cache); chunk token i
// of sequence s sits at position p = seq_lens[s] - C_s + i and attends to the
// cached tokens t <= p through the block table.
//
// Unit: (sequence, kv head, 128 query rows); a row is a (chunk token, q head
// of the kv head's group) pair, so one K/V tile serves all g heads of every
// token in the unit.  A CTA takes two adjacent units of one (sequence, kv
// head) -- they read the same K/V tiles -- and keeps the tensor core busy on
// one unit while the other runs its softmax:
//   - warp 17 (one lane) copies the units' q rows and then, through the
//     block table, each 64-token K and V tile with TMA into the 128-byte
//     swizzled layout the tensor core reads (3-stage K and V rings);
//   - warp 16 (one lane) owns tensor memory and issues, per tile,
//     O_0 += P_0 V, S_0' = Q_0 K'^T, O_1 += P_1 V, S_1' = Q_1 K'^T
//     (tcgen05.mma, M = 128 rows, fp32 accumulators in tensor memory);
//   - warps 0-7 and 8-15 are the two units' softmax groups, two threads per
//     row (one per half of the 64 scores and of the head_dim outputs): load
//     S from tensor memory, mask, exponentiate against a reference maximum,
//     write P back to tensor memory, where the P V product reads it as its
//     A operand (bf16 as hi + lo parts, so P V keeps fp32-level accuracy).
//     O stays in tensor memory across tiles; it is rescaled only when a
//     row's maximum passes its reference by 2^8.
// A unit without a partner (a decode row, the first row tile of a sequence
// with an odd count) splits its tiles instead: group 0 takes the even tiles,
// group 1 the odd ones, and group 0 merges the two partial (max, sum, O)
// results at the end.
// Every hand-off is an mbarrier; every wait is bounded (0.2 s of
// %globaltimer): a timeout sets PKV_DEVERR_TIMEOUT, every role leaves its
// loop, the copies and products already issued are drained, and the CTA
// frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <type_traits>

#include "pkv_device.cuh"
#include "pkv_internal.h"
#include "tcgen05.cuh"

namespace pkv {
namespace {

using namespace tc;

constexpr int kPfRows = 128;        // query rows per unit (tensor-core M)
constexpr int kPfTok = 64;          // KV tokens per tile (N of S, K of P V)
constexpr int kPfGroup = 256;       // softmax threads per unit: two per row
constexpr int kPfMmaWarp = 16;      // issues the tensor-core products, owns tensor memory
constexpr int kPfLoadWarp = 17;     // issues the TMA copies
constexpr int kPfThreads = 18 * 32;
constexpr int kPfStages = 3;        // K and V ring depth
constexpr int kPfTmemCols = 512;    // unit u: S in columns 256 u + [0, 64), O from 256 u + 64,
constexpr int kPfTmemP = 192;       //   P (hi, lo: 32 columns each) from 256 (1 - u) + 192: the
                                    //   other half from its O (measured 1 % faster than beside it)
constexpr uint64_t kPfWaitNs = 200000000ull;

// mbarriers
enum : int {
    kBarQ = 0,                             // q rows landed (TMA transaction count)
    kBarKFull = 1,                         // [stage] K tile landed
    kBarVFull = kBarKFull + kPfStages,     // [stage] V tile landed
    kBarKEmpty = kBarVFull + kPfStages,    // [stage] every S product of the K stage finished
    kBarVEmpty = kBarKEmpty + kPfStages,   // [stage] every P V product of the V stage finished
    kBarVFix = kBarVEmpty + kPfStages,     // the last V tile's rows past the unit's end are zeroed
    kBarS = kBarVFix + 1,                  // [unit] S ready
    kBarP = kBarS + 2,                     // [unit] P written (and S read): kPfGroup arrivals
    kBarO = kBarP + 2,                     // [unit] P V finished
    kBarDrain = kBarO + 2,                 // products drained (abort path)
    kNumBars = kBarDrain + 1
};

struct PrefillParams {
    void* out;
    const int32_t* tables;
    const int32_t* seq_lens;
    const int32_t* qstart;
    int* err;
    int64_t num_blocks;
    int num_seqs, num_heads, num_kv_heads, g, mbps, bs;
    float scale_log2;
    uint64_t wait_ns;  // limit of every wait (kPfWaitNs)
    int stop_tile;     // < 0; a test of the timeout path sets k >= 0: K/V tiles k, k+1, ... are never copied
};

// Named barrier over one softmax group (kPfGroup threads, whole warps) that
// also ORs a flag across it.
__device__ __forceinline__ bool group_sync_or(int id, bool flag) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}\n"
                 : "=r"(r) : "r"((uint32_t)flag), "r"(id), "n"(kPfGroup) : "memory");
    return r != 0;
}
// The same over both softmax groups (barrier 3, 2 kPfGroup threads).
__device__ __forceinline__ bool pair_sync_or(bool flag) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 3, %2, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}\n"
                 : "=r"(r) : "r"((uint32_t)flag), "n"(2 * kPfGroup) : "memory");
    return r != 0;
}
template <typename T, int D>
struct PfSmem {
    static constexpr int kQ = kPfRows * D * 2;     // one unit's q rows
    static constexpr int kTile = kPfTok * D * 2;   // one K or V tile
    static constexpr int kParts = std::is_same<T, __nv_bfloat16>::value ? 2 : 1;  // P hi (+ lo)
    static constexpr int kData = 2 * kQ + 2 * kPfStages * kTile + 1024;           // + alignment
    // at least 120 KB, so one CTA (and its 512 tensor-memory columns) per SM
    static constexpr int kBytes = kData > 120 * 1024 ? kData : 120 * 1024;
};

// The geometry of one 128-row unit.
struct PfUnit {
    int tok0, ntok, pos0, kv_end, nkv;
};

template <typename T, int D>
__global__ void __launch_bounds__(kPfThreads, 1)
pkv_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v) {
    using SM = PfSmem<T, D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int CH = D / 8;  // 16-byte chunks per row
    extern __shared__ uint8_t pf_raw[];
    uint8_t* sm = pf_raw + ((1024 - (smem_u32(pf_raw) & 1023)) & 1023);  // 1024-byte aligned operands
    uint8_t* qsm = sm;                          // [2 units]
    uint8_t* ksm = qsm + 2 * SM::kQ;            // [stage]
    uint8_t* vsm = ksm + kPfStages * SM::kTile; // [stage]
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ float xmax[2][2][2][kPfRows];    // [unit][tile parity][half][row] partial row maxima
    __shared__ float xsum[2][2][kPfRows];       // [group][half][row] partial row sums
    __shared__ float xref[kPfRows];             // group 1's reference maxima (split unit)
    volatile int* abort = &abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    // K/V tile kt sits in ring stage kt % kPfStages; its full / empty
    // barriers complete once per pass of the ring
    auto stg = [](int kt) { return kt % kPfStages; };
    auto pass = [](int kt) { return (uint32_t)((kt / kPfStages) & 1); };

    // ---- the unit pair: kv head from the block index, then pair u among all
    // sequences' pairs (warp-parallel scan; every warp finds it).  A
    // sequence's row tiles pair from the last: (n-1, n-2), (n-3, n-4), ...
    const int kh = (int)(blockIdx.x % p.num_kv_heads);
    const int64_t u = blockIdx.x / p.num_kv_heads;
    int s = -1, jp = 0, nrt_s = 0;
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
            const int npr = (nrt + 1) >> 1;
            int incl = npr;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            const int64_t lo = base + incl - npr;
            const unsigned hit = __ballot_sync(kFull, npr > 0 && u >= lo && u < lo + npr);
            if (hit) {
                const int src = __ffs(hit) - 1;
                s = s0 + src;
                const int64_t l0 = __shfl_sync(kFull, lo, src);
                nrt_s = __shfl_sync(kFull, nrt, src);
                jp = (int)(u - l0);  // a sequence's heaviest pair first
            }
            base += __shfl_sync(kFull, incl, 31);
        }
    }
    if (s < 0) return;  // past the last pair
    const int q0 = __ldg(p.qstart + s);
    const int C = __ldg(p.qstart + s + 1) - q0;
    const int L = __ldg(p.seq_lens + s);
    if (L < C || L > p.mbps * p.bs) {
        if (tid == 0) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
        return;
    }
    const int ctx = L - C;
    const int tpu = kPfRows / p.g;  // chunk tokens per unit (g divides 16)
    const int j0 = nrt_s - 1 - 2 * jp, j1 = j0 - 1;
    const int nunits = j1 >= 0 ? 2 : 1;
    auto make_unit = [&](int j) {
        PfUnit w;
        w.tok0 = j * tpu;
        w.ntok = min(tpu, C - w.tok0);
        w.pos0 = ctx + w.tok0;
        w.kv_end = w.pos0 + w.ntok;
        w.nkv = (w.kv_end + kPfTok - 1) / kPfTok;
        return w;
    };
    const PfUnit U0 = make_unit(j0);                 // the later rows: the longer K/V range
    const PfUnit U1 = make_unit(j1 >= 0 ? j1 : j0);  // (unused when nunits == 1)
    const int nkv = U0.nkv;
    // a unit alone splits its K/V tiles between the two groups (even / odd
    // tiles), whose partial results are merged at the end
    const bool split = nunits == 1;
    const bool need_fix = (U0.kv_end % kPfTok) != 0;  // V rows past the end must read as zeros

    // ---- tensor memory, barriers
    if (warp == kPfMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(kPfTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == kBarP || i == kBarP + 1) ? kPfGroup : 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = tmem_base;

    if (warp < 2 * (kPfGroup / 32)) {
        // ================= softmax group X: unit X (or, for a unit alone,
        // its tiles of stage X), two threads per row
        const int X = warp >> 3;
        {
            const PfUnit U = X && !split ? U1 : U0;
            const int kt0 = split ? X : 0, kstep = split ? 2 : 1;  // this group's tiles
            const int ntiles = split ? (nkv - X + 1) / 2 : U.nkv;
            const int wq = warp & 3, half = (warp >> 2) & 1;
            const int row = wq * 32 + lane;
            const int pos = (row / p.g < U.ntok) ? U.pos0 + row / p.g : -1;
            const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
            const uint32_t tS = tmem + lane_addr + X * 256 + half * (kPfTok / 2);
            const uint32_t tO = tmem + lane_addr + X * 256 + kPfTok + half * (D / 2);
            const uint32_t tP = tmem + lane_addr + (X ^ 1) * 256 + kPfTmemP + half * (kPfTok / 4);
            const float sl2 = p.scale_log2;
            float mref = -INFINITY, l = 0.f;  // reference maximum (log2 domain) and this half's sum
            bool failed = false;
#pragma unroll 1
            for (int i = 0; i < ntiles; ++i) {
                const int kt = kt0 + i * kstep;
                bool ok = !failed && mbar_wait(bar(kBarS + X), i & 1, abort, p.wait_ns);
                ok = __all_sync(kFull, ok);
                float sc[kPfTok / 2];
                float pm = -INFINITY;
                if (ok) {
                    tc_after_sync();
                    tc_ld32(tS, sc);
                    if (kt * kPfTok + kPfTok - 1 > U.pos0) {  // a tile on the causal diagonal
                        const int t0 = kt * kPfTok + half * (kPfTok / 2);
#pragma unroll
                        for (int c = 0; c < kPfTok / 2; ++c) sc[c] = t0 + c <= pos ? sc[c] : -INFINITY;
                    }
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c = 0; c < kPfTok / 2; ++c) m4[c & 3] = fmaxf(m4[c & 3], sc[c]);
                    pm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                }
                xmax[X][i & 1][half][row] = pm;
                if (group_sync_or(1 + X, !ok)) {
                    failed = true;
                    break;
                }
                // the row maximum of this tile (both halves), in the log2 domain
                const float mx = fmaxf(xmax[X][i & 1][0][row], xmax[X][i & 1][1][row]) * sl2;
                const bool grow = mx > mref + 8.f;  // also the first finite maximum
                float alpha = 1.f;
                if (grow) {
                    alpha = ex2(mref - mx);  // 0 while nothing was attended
                    l *= alpha;
                    mref = mx;
                }
                const float ref = mref == -INFINITY ? 0.f : mref;
                float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < kPfTok / 2; ++c) {
                    sc[c] = ex2(fmaf(sc[c], sl2, -ref));
                    ls4[c & 3] += sc[c];
                }
                l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
                if (i > 0) {  // P V of the previous tile done: its P buffer is free, O is settled
                    ok = mbar_wait(bar(kBarO + X), (i - 1) & 1, abort, p.wait_ns);
                    ok = __all_sync(kFull, ok);
                    if (ok) {
                        tc_after_sync();
                        if (__any_sync(kFull, grow)) {  // rescale this half row of O
#pragma unroll 1
                            for (int c0 = 0; c0 < D / 2; c0 += 16) {
                                float v[16];
                                tc_ld16(tO + c0, v);
#pragma unroll
                                for (int e = 0; e < 16; ++e) v[e] *= alpha;
                                tc_st16(tO + c0, v);
                            }
                        }
                    }
                }
                if (!ok) {
                    failed = true;
                    continue;  // the next tile's group barrier ends the loop for the whole group
                }
                // ---- this half of P into tensor memory: row = lane, two
                // tokens per 32-bit column (bf16 as hi + lo parts, 32 columns apart)
                {
                    uint32_t h[kPfTok / 4], lo[kPfTok / 4];
#pragma unroll
                    for (int e = 0; e < kPfTok / 4; ++e) {
                        const float a = sc[2 * e], b = sc[2 * e + 1];
                        h[e] = pack2<kBf16>(a, b);
                        if constexpr (kBf16) {
                            const float2 hf = unpack2<true>(h[e]);
                            lo[e] = pack2<true>(a - hf.x, b - hf.y);
                        }
                    }
                    tc_st16u(tP, h);
                    if constexpr (kBf16) tc_st16u(tP + kPfTok / 2, lo);
                    tc_wait_st();
                }
                tc_before_sync();
                mbar_arrive(bar(kBarP + X));
            }
            // ---- the last P V, then normalise (the halves' sums combined; a
            // split unit also merges group 1's partial result) and store
            bool ok = !failed && (ntiles == 0 || mbar_wait(bar(kBarO + X), (ntiles - 1) & 1, abort, p.wait_ns));
            // (group 1's last P V, read in the merge: after group 0's own last
            // one, at most that phase of group 1 is outstanding)
            if (split && X == 0 && nkv > 1) ok = ok && mbar_wait(bar(kBarO + 1), ((nkv >> 1) - 1) & 1, abort, p.wait_ns);
            ok = __all_sync(kFull, ok);
            xsum[X][half][row] = l;
            if (split && X == 1 && half == 0) xref[row] = mref;
            const bool bad = split ? pair_sync_or(!ok) : group_sync_or(1 + X, !ok);
            if (!bad && !(split && X == 1)) {
                tc_after_sync();
                float lt = xsum[X][0][row] + xsum[X][1][row];
                float a0 = 1.f, a1 = 0.f;
                const bool merge = split && nkv > 1;
                if (merge) {
                    const float m1 = xref[row], m = fmaxf(mref, m1);
                    a0 = mref == -INFINITY ? 0.f : ex2(mref - m);
                    a1 = m1 == -INFINITY ? 0.f : ex2(m1 - m);
                    lt = a0 * lt + a1 * (xsum[1][0][row] + xsum[1][1][row]);
                }
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
                a0 *= inv;
                a1 *= inv;
                T* out = static_cast<T*>(p.out) +
                         ((int64_t)(q0 + U.tok0 + row / p.g) * p.num_heads + (int64_t)kh * p.g + row % p.g) * D +
                         half * (D / 2);
#pragma unroll 1
                for (int c0 = 0; c0 < D / 2; c0 += 16) {
                    float v[16];
                    tc_ld16(tO + c0, v);  // every lane loads (warp-collective); only real rows store
                    if (merge) {
                        float v1[16];
                        tc_ld16(tO + 256 + c0, v1);  // group 1's O: same lanes, the next 256 columns
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = a0 * v[e] + a1 * v1[e];
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= a0;
                    }
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) w[e] = pack2<kBf16>(v[2 * e], v[2 * e + 1]);
                    if (pos >= 0) {
                        *reinterpret_cast<uint4*>(out + c0) = make_uint4(w[0], w[1], w[2], w[3]);
                        *reinterpret_cast<uint4*>(out + c0 + 8) = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
        }
    } else if (warp == kPfMmaWarp) {
        // ================= tensor-core issue (one lane)
        if (lane == 0) {
            const uint32_t id_s = tc_idesc<kBf16>(kPfRows, kPfTok, 0);
            const uint32_t id_o = tc_idesc<kBf16>(kPfRows, D, 1);
            // operand descriptors built once; per product only a constant
            // offset is added (the issue rate of this one thread bounds the
            // tensor core otherwise)
            const uint64_t dq0 = tc_desc(smem_u32(qsm), 16, 1024);
            const uint64_t dq1 = tc_desc(smem_u32(qsm + (split ? 0 : SM::kQ)), 16, 1024);
            const uint64_t dk0 = tc_desc(smem_u32(ksm), 16, 1024);
            const uint64_t dv0 = tc_desc(smem_u32(vsm), kPfTok * 128, 1024);
            auto issue_s = [&](int X, int st) {  // S_X = Q_X K^T (a split unit: both groups read q slot 0)
                const uint64_t qd = X ? dq1 : dq0;
                const uint64_t kd = desc_add(dk0, (uint32_t)(st * (SM::kTile >> 4)));
                const uint32_t d = tmem + X * 256;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc_mma(d, desc_add(qd, ((kk >> 2) * kPfRows * 128 + (kk & 3) * 32) >> 4),
                           desc_add(kd, ((kk >> 2) * kPfTok * 128 + (kk & 3) * 32) >> 4), id_s, kk > 0);
                tc_commit(bar(kBarS + X));
            };
            auto issue_pv = [&](int X, int st, bool acc) {  // O_X (+)= P_X V (hi, then lo; P in tensor memory)
                const uint64_t vd = desc_add(dv0, (uint32_t)(st * (SM::kTile >> 4)));
                const uint32_t d = tmem + X * 256 + kPfTok, a = tmem + (X ^ 1) * 256 + kPfTmemP;
#pragma unroll
                for (int part = 0; part < SM::kParts; ++part)
#pragma unroll
                    for (int kk = 0; kk < kPfTok / 16; ++kk)
                        tc_mma_ts(d, a + part * (kPfTok / 2) + kk * 8, desc_add(vd, (kk * 2048) >> 4), id_o,
                                  (acc || part > 0 || kk > 0) ? 1u : 0u);
                tc_commit(bar(kBarO + X));
            };
            bool ok = mbar_wait(bar(kBarQ), 0, abort, p.wait_ns);
            if (!split) {
                // paired units: every tile serves both; per tile
                // O_0 += P_0 V, S_0' = Q_0 K'^T, O_1 += P_1 V, S_1' = Q_1 K'^T
                ok = ok && mbar_wait(bar(kBarKFull), 0, abort, p.wait_ns);
                if (ok) {
                    tc_after_sync();
                    issue_s(0, 0);
                    issue_s(1, 0);
                    tc_commit(bar(kBarKEmpty));
                }
#pragma unroll 1
                for (int kt = 0; ok && kt < nkv; ++kt) {
                    const int st = stg(kt), sn = stg(kt + 1);
                    const bool a1 = kt < U1.nkv, a1n = kt + 1 < U1.nkv;
                    ok = mbar_wait(bar(kBarVFull + st), pass(kt), abort, p.wait_ns) &&
                         (kt != nkv - 1 || !need_fix || mbar_wait(bar(kBarVFix), 0, abort, p.wait_ns)) &&
                         mbar_wait(bar(kBarP), kt & 1, abort, p.wait_ns);
                    if (!ok) break;
                    tc_after_sync();
                    issue_pv(0, st, kt > 0);
                    if (!a1) tc_commit(bar(kBarVEmpty + st));
                    if (kt + 1 < nkv) {
                        ok = mbar_wait(bar(kBarKFull + sn), pass(kt + 1), abort, p.wait_ns);
                        if (!ok) break;
                        tc_after_sync();
                        issue_s(0, sn);
                        if (!a1n) tc_commit(bar(kBarKEmpty + sn));
                    }
                    if (a1) {
                        ok = mbar_wait(bar(kBarP + 1), kt & 1, abort, p.wait_ns);
                        if (!ok) break;
                        tc_after_sync();
                        issue_pv(1, st, kt > 0);
                        tc_commit(bar(kBarVEmpty + st));
                        if (a1n) {
                            issue_s(1, sn);
                            tc_commit(bar(kBarKEmpty + sn));
                        }
                    }
                }
            } else {
                // a split unit: group X takes tiles 2 i + X; per step i:
                // O_0 += P_0 V_2i, S_0 = Q K_2i+2^T, O_1 += P_1 V_2i+1, S_1 = Q K_2i+3^T
#pragma unroll 1
                for (int X = 0; ok && X < 2 && X < nkv; ++X) {
                    ok = mbar_wait(bar(kBarKFull + stg(X)), pass(X), abort, p.wait_ns);
                    if (!ok) break;
                    tc_after_sync();
                    issue_s(X, stg(X));
                    tc_commit(bar(kBarKEmpty + stg(X)));
                }
#pragma unroll 1
                for (int i = 0; ok && 2 * i < nkv; ++i) {
#pragma unroll 1
                    for (int X = 0; X < 2; ++X) {
                        const int kt = 2 * i + X;
                        if (kt >= nkv) break;
                        ok = mbar_wait(bar(kBarVFull + stg(kt)), pass(kt), abort, p.wait_ns) &&
                             (kt != nkv - 1 || !need_fix || mbar_wait(bar(kBarVFix), 0, abort, p.wait_ns)) &&
                             mbar_wait(bar(kBarP + X), i & 1, abort, p.wait_ns);
                        if (!ok) break;
                        tc_after_sync();
                        issue_pv(X, stg(kt), i > 0);
                        tc_commit(bar(kBarVEmpty + stg(kt)));
                        if (kt + 2 < nkv) {
                            ok = mbar_wait(bar(kBarKFull + stg(kt + 2)), pass(kt + 2), abort, p.wait_ns);
                            if (!ok) break;
                            tc_after_sync();
                            issue_s(X, stg(kt + 2));
                            tc_commit(bar(kBarKEmpty + stg(kt + 2)));
                        }
                    }
                }
            }
            tc_commit(bar(kBarDrain));  // every product issued has finished before tensor memory is freed
            mbar_wait(bar(kBarDrain), 0, nullptr, p.wait_ns);
        }
        __syncwarp();
    } else if (warp == kPfLoadWarp) {
        // ================= TMA copies (one lane), then the V tail fix (the warp)
        bool ok = true;
        if (lane == 0) {
            int nk[kPfStages] = {}, nv[kPfStages] = {};
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_v)) : "memory");
            mbar_expect_tx(bar(kBarQ), (uint32_t)(nunits * SM::kQ));
#pragma unroll 1
            for (int X = 0; X < nunits; ++X) {
                const PfUnit& W = X ? U1 : U0;
#pragma unroll
                for (int cb = 0; cb < D / 64; ++cb)
                    tma_load3(smem_u32(qsm + X * SM::kQ + cb * kPfRows * 128), &tmap_q, cb * 64, kh * p.g,
                              q0 + W.tok0, bar(kBarQ));
            }
            const int32_t* trow = p.tables + (int64_t)s * p.mbps;
            const int lg_bs = p.bs == 16 ? 4 : 5;
            const int nblk = kPfTok >> lg_bs;
            const int kt_end = p.stop_tile < 0 ? nkv : min(nkv, p.stop_tile);
#pragma unroll 1
            for (int kt = 0; kt < kt_end; ++kt) {
                const int st = stg(kt);
                int phys[kPfTok / 16];
                int nb = 0;
#pragma unroll
                for (int jb = 0; jb < kPfTok / 16; ++jb) {
                    const int t = kt * kPfTok + (jb << lg_bs);
                    phys[jb] = 0;
                    if (jb < nblk && t < U0.kv_end) {
                        int ph = __ldg(trow + (t >> lg_bs));
                        if (ph < 0 || ph >= p.num_blocks) {
                            raise_error(p.err, PKV_DEVERR_BLOCK_ID);
                            ph = 0;
                        }
                        phys[jb] = ph;
                        ++nb;
                    }
                }
                const uint32_t bytes = (uint32_t)(nb * p.bs * D * 2);
                if (kt >= kPfStages && !(ok = mbar_wait(bar(kBarKEmpty + st), pass(kt - kPfStages), abort, p.wait_ns))) break;
                mbar_expect_tx(bar(kBarKFull + st), bytes);
#pragma unroll 1
                for (int jb = 0; jb < nb; ++jb)
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load3(smem_u32(ksm + st * SM::kTile + cb * kPfTok * 128 + jb * p.bs * 128), &tmap_k,
                                  cb * 64, kh, phys[jb] * p.bs, bar(kBarKFull + st));
                ++nk[st];
                if (kt >= kPfStages && !(ok = mbar_wait(bar(kBarVEmpty + st), pass(kt - kPfStages), abort, p.wait_ns))) break;
                mbar_expect_tx(bar(kBarVFull + st), bytes);
#pragma unroll 1
                for (int jb = 0; jb < nb; ++jb)
#pragma unroll
                    for (int cb = 0; cb < D / 64; ++cb)
                        tma_load3(smem_u32(vsm + st * SM::kTile + cb * kPfTok * 128 + jb * p.bs * 128), &tmap_v,
                                  cb * 64, kh, phys[jb] * p.bs, bar(kBarVFull + st));
                ++nv[st];
            }
            if (kt_end < nkv) ok = false;  // (timeout test) the other roles wait for the missing tiles
            if (!ok) {  // let the copies in flight land before the CTA ends
                mbar_wait(bar(kBarQ), 0, nullptr, p.wait_ns);
                for (int st = 0; st < kPfStages; ++st) {
                    if (nk[st]) mbar_wait(bar(kBarKFull + st), (nk[st] - 1) & 1, nullptr, p.wait_ns);
                    if (nv[st]) mbar_wait(bar(kBarVFull + st), (nv[st] - 1) & 1, nullptr, p.wait_ns);
                }
            }
        }
        __syncwarp();
        ok = __shfl_sync(kFull, ok, 0);
        if (need_fix) {  // zero the last V tile's rows at and past the unit's end
            const int kl = nkv - 1, st = stg(kl);
            bool fine = ok && mbar_wait(bar(kBarVFull + st), pass(kl), abort, p.wait_ns);
            fine = __all_sync(kFull, fine);
            if (fine) {
                const int r0 = U0.kv_end - kl * kPfTok;
                uint8_t* vt = vsm + st * SM::kTile;
                for (int i = lane; i < (kPfTok - r0) * CH; i += 32)
                    *reinterpret_cast<uint4*>(vt + tc_off(r0 + i / CH, i % CH, kPfTok)) = make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(kBarVFix));
            }
        }
    }

    tc_before_sync();
    __syncthreads();
    if (warp == kPfMmaWarp) {
        tc_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kPfTmemCols));
    }
    if (tid == 0 && abort_flag) raise_error(p.err, PKV_DEVERR_TIMEOUT);
}

template <typename T, int D>
pkv_status launch_prefill(const PrefillParams& p, const void* query, const void* kc, const void* vc,
                          int64_t num_tokens, int64_t num_blocks, int64_t grid, cudaStream_t st) {
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr int kSmem = PfSmem<T, D>::kBytes;
    static_assert(kSmem <= 227 * 1024 - 8 * 1024, "prefill shared memory");
    CUtensorMap tq, tk, tv;
    pkv_status r = encode_map(&tq, kBf16, query, D, p.num_heads, num_tokens, p.g, kPfRows / p.g);
    if (r == PKV_OK) r = encode_map(&tk, kBf16, kc, D, p.num_kv_heads, num_blocks * p.bs, 1, p.bs);
    if (r == PKV_OK) r = encode_map(&tv, kBf16, vc, D, p.num_kv_heads, num_blocks * p.bs, 1, p.bs);
    if (r != PKV_OK) return r;
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
    pkv_prefill_kernel<T, D><<<(unsigned)grid, kPfThreads, kSmem, st>>>(p, tq, tk, tv);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ECUDA, "prefill launch: %s", cudaGetErrorString(e));
    return PKV_OK;
}

// A timeout test armed by pkv_testing_prefill_timeout for the next
// pkv_paged_prefill call on this thread (stop_tile < 0: not armed).
thread_local int t_test_stop_tile = -1;
thread_local uint64_t t_test_wait_ns = 0;

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_testing_prefill_timeout(int stop_tile, uint64_t wait_ns) {
    if (stop_tile < 0) return fail(PKV_EINVAL, "stop_tile < 0");
    if (wait_ns < 100000ull || wait_ns > kPfWaitNs)
        return fail(PKV_EINVAL, "wait_ns outside [1e5, %llu]", (unsigned long long)kPfWaitNs);
    t_test_stop_tile = stop_tile;
    t_test_wait_ns = wait_ns;
    return PKV_OK;
}

extern "C" pkv_status pkv_paged_prefill(void* out, const void* query, pkv_dtype q_dtype,
                                        const void* key_cache, const void* value_cache,
                                        pkv_dtype cache_dtype, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* seq_lens,
                                        const int32_t* query_start, int num_seqs,
                                        int64_t num_query_tokens, int num_heads, int num_kv_heads,
                                        int head_dim, int block_size, int64_t num_blocks, float scale,
                                        pkv_stream_t stream) {
    // a timeout test applies to this call only, whatever it returns
    const int stop_tile = t_test_stop_tile;
    const uint64_t wait_ns = t_test_wait_ns ? t_test_wait_ns : kPfWaitNs;
    t_test_stop_tile = -1;
    t_test_wait_ns = 0;
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
    p.wait_ns = wait_ns;
    p.stop_tile = stop_tile;
    // unit pairs: sum_s ceil(ceil(C_s g / 128) / 2) <= ceil(T g / 256) + S
    const int64_t pairs = (num_query_tokens * g + 2 * kPfRows - 1) / (2 * kPfRows) + num_seqs;
    const int64_t grid = pairs * num_kv_heads;
    if (grid > 0x7fffffffLL) return fail(PKV_EUNSUPPORTED, "too many query rows");
    // TMA coordinates are 32-bit: token rows of the query and of the pool
    if (num_query_tokens > 0x7fffffffLL || num_blocks * block_size > 0x7fffffffLL)
        return fail(PKV_EUNSUPPORTED, "query or pool too large for 32-bit copy coordinates");
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int64_t T = num_query_tokens;
    if (cache_dtype == PKV_F16)
        return head_dim == 64
                   ? launch_prefill<__half, 64>(p, query, key_cache, value_cache, T, num_blocks, grid, cs)
                   : launch_prefill<__half, 128>(p, query, key_cache, value_cache, T, num_blocks, grid, cs);
    return head_dim == 64
               ? launch_prefill<__nv_bfloat16, 64>(p, query, key_cache, value_cache, T, num_blocks, grid, cs)
               : launch_prefill<__nv_bfloat16, 128>(p, query, key_cache, value_cache, T, num_blocks, grid, cs);
}
