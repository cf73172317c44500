// cascade_tc.cuh -- the cascade prefix pass on the 5th-generation tensor core
// (tcgen05).  The shared prefix of a group (zwxr.cn section 3.4: blocks shared
// copy-on-write by the members of a parallel-sampling or beam group) is read
// once per (group, kv head) and serves every member's query rows: the rows
// are few (members x q heads of the kv head, at most 32 here), the tokens
// many, so the tokens are the tensor core's M dimension:
//   S^T [128 tokens x 32 rows] = K_tile [128 x D] . Q^T         (A: K tile, B: q rows)
//   O^T [D x 32 rows]         += V_tile^T [D x 128] . P^T       (A: V tile read MN-major, B: P^T)
// with fp32 accumulators in tensor memory.  Per CTA (one per SM), over an
// equal contiguous range of 128-token tiles of all units (stream-K; a unit
// split between CTAs leaves segments that the combine pass merges):
//   - warps 5-8 gather each K and V tile through the group's block table
//     (two warps per tile, 64 rows each) with 16-byte cp.async copies
//     straight into the 128-byte-swizzled operand layout (2-stage rings;
//     rows past the prefix zero-filled; each lane's copies arrive on the
//     tile's full barrier as they complete, and the issuing thread fences
//     them to the tensor core's proxy), and warp 5 copies a unit's q rows;
//   - warp 4 (one lane) issues S^T of tile n and then O^T += V^T P^T of tile
//     n-1, so the softmax of one tile runs beside the products of the next;
//   - warps 0-3 (thread = token for S^T, = head_dim index for O^T) mask and
//     scale the scores, take each row's maximum across the 128 tokens
//     (a warp reduce-scatter, then the four warps through shared memory),
//     exponentiate against a reference maximum that moves only when a row's
//     maximum passes it by 2^8 (then l and O^T are rescaled), and write P^T
//     as bf16 / f16 hi + lo parts into shared memory for the next product.
// The result is the prefix partial (m, l, o) of every member row, exactly as
// the mma.sync prefix pass writes it.  Every wait is bounded; a timeout sets
// PKV_DEVERR_TIMEOUT and every role leaves.
#pragma once

#include "cascade.cuh"
#include "tcgen05.cuh"

namespace pkv {

constexpr int kTcTok = 128;            // prefix tokens per K/V tile (M of S^T, K of O^T)
constexpr int kTcRows = 32;            // member rows per unit (N); missing rows are zero
constexpr int kTcD = 128;              // head_dim (M of O^T)
constexpr int kTcKStages = 2;          // K ring depth (a slot frees when S^T of its tile finishes)
constexpr int kTcVStages = 2;          // V ring depth (a slot frees only after the tile's O^T product;
                                       // 3 stages measured no faster)
constexpr int kTcMmaWarp = 4;
constexpr int kTcLoadWarp0 = 5;        // warps 5-6: K tile halves (and q rows); 7-8: V tile halves
constexpr int kTcThreads = 9 * 32;
// Tensor memory: S^T buffers at columns 0 and 32; O^T at 64.  With bf16
// caches P^T's hi and lo parts are stacked as the 64 rows of one operand, so
// each O^T product has N = 64 (half the products of two N = 32 parts) and
// O^T's columns 64 + r (hi) and 96 + r (lo) sum to row r's output.
constexpr int kTcTmemCols = 128;
constexpr int kTcTile = kTcTok * kTcD * 2;       // one K or V tile: 32 KB
constexpr int kTcQ = kTcRows * kTcD * 2;         // one unit's q rows: 8 KB
constexpr int kTcP = kTcRows * kTcTok * 2;       // one P^T part: 8 KB
constexpr int kTcSmem = (kTcKStages + kTcVStages) * kTcTile + 2 * kTcQ + 2 * 2 * kTcP + 1024;
static_assert(kTcSmem <= 227 * 1024, "shared memory budget");
constexpr uint64_t kTcWaitNs = 200000000ull;     // limit of every wait (0.2 s)

enum : int {
    kTbKFull = 0,                          // [stage] K tile landed (64 copy-lane arrivals)
    kTbVFull = kTbKFull + kTcKStages,      // [stage] V tile landed
    kTbKEmpty = kTbVFull + kTcVStages,     // [stage] S^T of the tile finished
    kTbVEmpty = kTbKEmpty + kTcKStages,    // [stage] O^T product of the tile finished
    kTbQFull = kTbVEmpty + kTcVStages,     // [q buffer] a unit's q rows written
    kTbQEmpty = kTbQFull + 2,              // [q buffer] the unit's last S^T finished
    kTbS = kTbQEmpty + 2,                  // [S buffer] S^T ready
    kTbP = kTbS + 2,                       // [P buffer] P^T written (128 arrivals)
    kTbO = kTbP + 2,                       // an O^T product finished (one phase per tile)
    kTbDrain = kTbO + 1,                   // products drained (abort path)
    kTbCount = kTbDrain + 1
};

// Reduce-scatter of 32 values per lane over the warp: afterwards v[0] of lane
// l is the reduction over all 32 lanes of their v[l] (max or sum).
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float keep = up ? v[i + o] : v[i];
            const float send = up ? v[i] : v[i + o];
            const float got = __shfl_xor_sync(kFull, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

// 32 fp32 columns into this thread's tensor-memory lane (asynchronous:
// tc::tc_wait_st before the columns are read again).
__device__ __forceinline__ void tc_st32(uint32_t taddr, const float* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                   "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                   "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
                   "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
                   "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
                   "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
                   "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
                   "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
                   "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
                   "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
                   "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
                 : "memory");
}

// Named barrier 1 over the four softmax warps that also ORs a flag across
// them: a decision every one of the 128 threads takes together.
__device__ __forceinline__ bool tc_group_or(bool flag) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}\n"
                 : "=r"(r) : "r"((uint32_t)flag) : "memory");
    return r != 0;
}

// Member rows of prefix unit j of group g: rows [R*rc, R*rc + R) of the
// group's members x q heads of kv head kh (row = member * g + head).
struct TcUnit {
    int s = -1, j = -1, kh, rc, nrows, o0, first_member;
    __device__ void locate(const DecodeParams& p, const CascadeParams& c, int g, int jj) {
        if (s == g && j == jj) return;
        s = g;
        j = jj;
        kh = jj / c.row_chunks;
        rc = jj % c.row_chunks;
        o0 = __ldg(c.grp_offsets + g);
        const int total = (__ldg(c.grp_offsets + g + 1) - o0) * p.g;
        nrows = max(0, min(kTcRows, total - kTcRows * rc));
        first_member = __ldg(c.grp_members + o0);
    }
};

template <typename T>
__global__ void __launch_bounds__(kTcThreads, 1)
pkv_prefix_tc_kernel(const DecodeParams p, const CascadeParams c) {
    using namespace tc;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    // launched as a programmatic dependent of the setup pass: its results
    // (prefix_eff, seq_start, member_info) are complete and visible only after
    // the wait; then the suffix pass may be scheduled (it reads seq_start)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t tc_raw[];
    uint8_t* sm = tc_raw + ((1024 - (smem_u32(tc_raw) & 1023)) & 1023);  // 1024-byte aligned operands
    uint8_t* ksm = sm;                               // [stage]
    uint8_t* vsm = ksm + kTcKStages * kTcTile;       // [stage]
    uint8_t* qsm = vsm + kTcVStages * kTcTile;       // [q buffer]
    uint8_t* psm = qsm + 2 * kTcQ;                   // [P buffer][part]
    __shared__ __align__(8) uint64_t bars[kTbCount];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;
    __shared__ float red[2][4][32];                  // [tile parity][warp][row] partial row maxima
    __shared__ float lred[4][32];                    // [warp][row] partial row sums
    volatile int* abort = &abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    if (tid == 0) {
        for (int i = 0; i < kTbCount; ++i) {
            const bool full = (i >= kTbKFull && i < kTbKFull + kTcKStages) || (i >= kTbVFull && i < kTbVFull + kTcVStages);
            const bool qfull = i == kTbQFull || i == kTbQFull + 1;
            mbar_init(bar(i), i == kTbP || i == kTbP + 1 ? 128 : full ? 64 : qfull ? 32 : 1);  // copy lanes arrive
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kTcMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base)),
                     "r"(kTcTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
    }
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = tmem_base;

    // every role walks the same tile range: units (group, kv head, row chunk)
    // of ceil(prefix / 128) tiles, laid end to end and cut in equal ranges
    const Lens<false> ln{c.prefix_eff, nullptr, c.num_groups, p.num_kv_heads * c.row_chunks, 0x7fffffff};
    int64_t workers = gridDim.x;
    const int64_t W = total_tiles<kTcTok>(ln);
    if (c.split_grid > 0) {
        // beside the suffix pass: this pass's share of the grid (the CTAs past
        // it find no tiles; they free their SMs for the suffix pass)
        const Lens<true> lsuf{p.seq_lens, c.seq_start, p.num_seqs, p.num_kv_heads * p.nch,
                              p.max_blocks_per_seq * p.block_size};
        workers = max(1, cascade_prefix_ctas(W, kTcTok, total_tiles<kTileTokens>(lsuf), kTileTokens, gridDim.x));
    }
    const int64_t chunk = (W + workers - 1) / workers;
    const int64_t tb = min(W, (int64_t)blockIdx.x * chunk), te = min(W, tb + chunk);
    const uint64_t lim = kTcWaitNs;
    constexpr int kParts = kBf16 ? 2 : 1;  // P^T as hi + lo bf16 parts, or one f16 part

    if (tb < te) {
        Walk<kTcTok> w;
        w.init(ln, tb, te);
        TcUnit u;
        if (warp >= kTcLoadWarp0) {
            // ================= copies: warps 5-6 the two 64-row halves of
            // each K tile (warp 5 also the q rows), warps 7-8 those of each V
            // tile.  16-byte cp.async per (row, chunk) into the 128-byte-
            // swizzled operand layout, rows past the prefix zero-filled;
            // every lane's copies of a tile arrive on its full barrier when
            // they complete (64 arrivals), so no warp waits for its copies.
            const int lw = warp - kTcLoadWarp0;
            const bool is_k = lw < 2;
            const int half = lw & 1;
            const uint8_t* cache = is_k ? p.key_cache : p.value_cache;
            uint8_t* ring = is_k ? ksm : vsm;
            const int full0 = is_k ? kTbKFull : kTbVFull, empty0 = is_k ? kTbKEmpty : kTbVEmpty;
            const int stages = is_k ? kTcKStages : kTcVStages;
            const int lg_bs = 31 - __clz(p.block_size);
            const int bs = 1 << lg_bs;
            const int bpt = kTcTok >> lg_bs;   // blocks per tile
            const int bph = bpt / 2;           // blocks per half (block sizes up to 64 tokens)
            const int64_t row_bytes = (int64_t)p.num_kv_heads * kTcD * 2;  // between tokens
            const int ch = lane & 15, r0 = lane >> 4;  // this lane: chunk ch of rows r0, r0 + 2, ...
            // swizzled chunk offsets of rows r0 + 2k (they repeat every 4 rows pairs)
            uint32_t so[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) so[k4] = (uint32_t)((((ch & 7) ^ ((r0 + 2 * k4) & 7)) << 4) + (r0 + 2 * k4) * 128);
            const uint32_t col = (uint32_t)((ch >> 3) * (kTcTok * 128));
            bool ok = true;
            for (int n = 0; ok && !w.done; ++n) {
                u.locate(p, c, w.s, w.j);
                const int st = n % stages;
                if (n >= stages)
                    ok = __all_sync(kFull, mbar_wait(bar(empty0 + st), (uint32_t)(((n / stages) & 1) ^ 1), abort, lim));
                if (!ok) break;
                if (lw == 0 && w.first()) {
                    // the unit's q rows into q buffer (ord & 1) first: cp.async
                    // of the rows' 16-byte chunks (rows past the group
                    // zero-filled), arriving on the q barrier as they complete
                    const int qb = w.ord & 1;
                    if (w.ord >= 2)
                        ok = __all_sync(kFull, mbar_wait(bar(kTbQEmpty + qb), (uint32_t)(((w.ord - 2) >> 1) & 1), abort, lim));
                    if (!ok) break;
                    const uint32_t q = smem_u32(qsm + qb * kTcQ);
                    constexpr int CPR = kTcD * 2 / 16;  // 16-byte chunks per row
                    const int row_l = kTcRows * u.rc + lane;  // lane l: the member of row l
                    const int mem_l = lane < u.nrows ? __ldg(c.grp_members + u.o0 + row_l / p.g) : 0;
#pragma unroll
                    for (int k = 0; k < kTcRows * CPR / 32; ++k) {
                        const int idx = lane + 32 * k, rr = idx / CPR, cc = idx % CPR;
                        const int sq = __shfl_sync(kFull, mem_l, rr);
                        const int row2 = kTcRows * u.rc + rr;  // member row within the group
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.q) +
                            (((int64_t)sq * p.num_heads + (int64_t)u.kh * p.g + row2 % p.g) * kTcD) * 2 + cc * 16;
                        cp_async16_zfill(q + tc_off(rr, cc, kTcRows), src, rr < u.nrows ? 16u : 0u);
                    }
                    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(kTbQFull + qb)) : "memory");
                }
                const int tok0 = w.i * kTcTok;
                const int nblk = (w.L + bs - 1) >> lg_bs;
                int phys = 0;
                if (lane < bph) {
                    const int b = (tok0 >> lg_bs) + half * bph + lane;
                    if (b < nblk) {
                        phys = __ldg(p.block_tables + (int64_t)u.first_member * p.max_blocks_per_seq + b);
                        if (phys < 0 || phys >= p.num_blocks) {
                            raise_error(p.err, PKV_DEVERR_BLOCK_ID);
                            phys = 0;
                        }
                    }
                }
                const uint32_t dst_t = smem_u32(ring + st * kTcTile) + col;
                const uint8_t* src_l = cache + (int64_t)u.kh * kTcD * 2 + ch * 16 + r0 * row_bytes;
                const int64_t step2 = 2 * row_bytes;
                const bool full_tile = tok0 + kTcTok <= w.L;
                for (int bb = 0; bb < bph; ++bb) {
                    const int b = half * bph + bb;  // block of the tile
                    const int pb = __shfl_sync(kFull, phys, bb);
                    const uint8_t* src = src_l + ((int64_t)pb << lg_bs) * row_bytes;
                    const uint32_t dst = dst_t + (uint32_t)((b << lg_bs) * 128);
                    if (full_tile) {
#pragma unroll 8
                        for (int k = 0; k < bs / 2; ++k)
                            cp_async16(dst + so[k & 3] + (k >> 2) * 1024, src + k * step2);
                    } else {
                        for (int k = 0; k < bs / 2; ++k) {
                            const int r = (b << lg_bs) + r0 + 2 * k;  // row (token) of the tile
                            cp_async16_zfill(dst + so[k & 3] + (k >> 2) * 1024, src + k * step2,
                                             tok0 + r < w.L ? 16u : 0u);
                        }
                    }
                }
                // each lane's copies arrive on the full barrier as they complete
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar(full0 + st)) : "memory");
                w.advance(ln);
            }
            // every copy in flight completes before the warp moves on
            cp_async_wait<0>();
            if (!ok) *abort = 1;
        } else if (warp == kTcMmaWarp) {
            // ================= tensor-core issue (one lane)
            const uint32_t id_s = tc_idesc<kBf16>(kTcTok, kTcRows, 0, 0);
            constexpr int kPvN = kParts * kTcRows;  // P^T rows: hi (and lo) parts stacked
            const uint32_t id_o = tc_idesc<kBf16>(kTcD, kPvN, 0, 1);
            const uint64_t dk0 = tc_desc(smem_u32(ksm), 16, 1024);
            const uint64_t dq0 = tc_desc(smem_u32(qsm), 16, 1024);
            const uint64_t dv0 = tc_desc(smem_u32(vsm), kTcTok * 128, 1024);
            const uint64_t dp0 = tc_desc(smem_u32(psm), 16, 1024);
            bool ok = true;
            int qb = 0;
            // O^T += V^T P^T of tile m (its first tile in this range overwrites)
            auto issue_pv = [&](int m, bool first) {
                const int st = m % kTcVStages;
                ok = ok && __all_sync(kFull, mbar_wait(bar(kTbP + (m & 1)), (uint32_t)((m >> 1) & 1), abort, lim));
                ok = ok && __all_sync(kFull, mbar_wait(bar(kTbVFull + st), (uint32_t)((m / kTcVStages) & 1), abort, lim));
                if (!ok) return;
                fence_async_smem();  // the cp.async-written V tile to the tensor core
                tc_after_sync();
                if (lane == 0) {
                    const uint64_t vd = desc_add(dv0, (uint32_t)(st * (kTcTile >> 4)));
                    const uint64_t pd = desc_add(dp0, (uint32_t)(((m & 1) * 2 * kTcP) >> 4));
#pragma unroll
                    for (int kk = 0; kk < kTcTok / 16; ++kk)
                        tc_mma(tmem + 64, desc_add(vd, (uint32_t)((kk * 2048) >> 4)),
                               desc_add(pd, (uint32_t)((((kk >> 2) * kPvN * 128) + (kk & 3) * 32) >> 4)), id_o,
                               (!first || kk > 0) ? 1u : 0u);
                    tc_commit(bar(kTbO));
                    tc_commit(bar(kTbVEmpty + st));
                }
                __syncwarp();
            };
            bool prev_first = false;
            int n = 0;
            for (; ok && !w.done; ++n) {
                const int st = n % kTcKStages;
                ok = __all_sync(kFull, mbar_wait(bar(kTbKFull + st), (uint32_t)((n / kTcKStages) & 1), abort, lim));
                const bool first = w.first();
                if (ok && first) {
                    qb = w.ord & 1;
                    ok = __all_sync(kFull, mbar_wait(bar(kTbQFull + qb), (uint32_t)((w.ord >> 1) & 1), abort, lim));
                }
                if (!ok) break;
                fence_async_smem();  // the cp.async-written K tile (and q rows) to the tensor core
                tc_after_sync();
                if (lane == 0) {
                    const uint64_t kd = desc_add(dk0, (uint32_t)(st * (kTcTile >> 4)));
                    const uint64_t qd = desc_add(dq0, (uint32_t)((qb * kTcQ) >> 4));
#pragma unroll
                    for (int kk = 0; kk < kTcD / 16; ++kk)
                        tc_mma(tmem + 32 * (n & 1), desc_add(kd, (uint32_t)((((kk >> 2) * kTcTok * 128) + (kk & 3) * 32) >> 4)),
                               desc_add(qd, (uint32_t)((((kk >> 2) * kTcRows * 128) + (kk & 3) * 32) >> 4)), id_s,
                               kk > 0 ? 1u : 0u);
                    tc_commit(bar(kTbS + (n & 1)));
                    tc_commit(bar(kTbKEmpty + st));
                    if (w.last()) tc_commit(bar(kTbQEmpty + qb));
                }
                __syncwarp();
                if (n > 0) issue_pv(n - 1, prev_first);
                prev_first = first;
                w.advance(ln);
            }
            if (ok && n > 0) issue_pv(n - 1, prev_first);
            if (!ok) {
                *abort = 1;
                // drain the products already issued before the memory is freed
                if (lane == 0) tc_commit(bar(kTbDrain));
                __syncwarp();
                mbar_wait(bar(kTbDrain), 0, nullptr, lim);
            }
        } else {
            // ================= softmax and output (warps 0-3, 128 threads)
            // Every decision to leave is taken by all 128 threads together
            // (tc_group_or), so no named barrier waits for a warp that left.
            const int t = tid;  // token of S^T, head_dim index of O^T
            const uint32_t lane_addr = (uint32_t)(32 * warp) << 16;
            float l[32], m_lane = -INFINITY;  // m_lane: lane r's reference maximum of row r
            int pv_seen = 0;                  // O^T products known finished
            bool failed = false;
            auto wait_pv = [&](int upto) {   // products of tiles < upto finished
                bool ok = true;
                while (ok && pv_seen < upto) {
                    ok = mbar_wait(bar(kTbO), (uint32_t)(pv_seen & 1), abort, lim);
                    ++pv_seen;
                }
                tc_after_sync();
                return ok;
            };
            for (int n = 0; !w.done; ++n) {
                if (w.first()) {
#pragma unroll
                    for (int r = 0; r < 32; ++r) l[r] = 0.f;
                    m_lane = -INFINITY;
                }
                const bool s_ok = mbar_wait(bar(kTbS + (n & 1)), (uint32_t)((n >> 1) & 1), abort, lim);
                if ((failed = tc_group_or(!s_ok))) break;
                tc_after_sync();
                float x[32];
                tc_ld32(tmem + lane_addr + 32 * (n & 1), x);
                const bool valid = w.i * kTcTok + t < w.L;
#pragma unroll
                for (int r = 0; r < 32; ++r) x[r] = valid ? x[r] * p.scale_log2 : -INFINITY;
                // row maxima over the 128 tokens
                float v[32];
#pragma unroll
                for (int r = 0; r < 32; ++r) v[r] = x[r];
                red[n & 1][warp][lane] = warp_reduce_scatter32<true>(v);
                asm volatile("bar.sync 1, 128;" ::: "memory");
                const float M = fmaxf(fmaxf(red[n & 1][0][lane], red[n & 1][1][lane]),
                                      fmaxf(red[n & 1][2][lane], red[n & 1][3][lane]));
                // lazy reference: moves (all rows at once) only when some
                // row's maximum passes it by more than 2^8; every warp takes
                // the same decision from the same maxima
                const bool grow = __any_sync(kFull, M > m_lane + 8.f);
                float a_lane = 1.f;
                if (grow) {
                    const float mn = fmaxf(m_lane, M);
                    a_lane = ex2(m_lane - mn);
                    m_lane = mn;
#pragma unroll
                    for (int r = 0; r < 32; ++r) l[r] *= __shfl_sync(kFull, a_lane, r);
                }
                // P^T (rows x tokens, K-major), bf16 as hi + lo parts, into
                // buffer n & 1 (its last reader, the product of tile n-2,
                // finished before S^T of tile n did)
                uint8_t* p0 = psm + (n & 1) * 2 * kTcP;  // rows [0, 32): hi; [32, 64): lo
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    const float e = ex2(x[r] - __shfl_sync(kFull, m_lane, r));
                    l[r] += e;
                    const uint32_t hb = pack2<kBf16>(e, 0.f) & 0xFFFFu;
                    *reinterpret_cast<uint16_t*>(p0 + tc_off(r, t >> 3, kParts * kTcRows) + (t & 7) * 2) = (uint16_t)hb;
                    if constexpr (kParts == 2) {
                        const float hi = unpack2<kBf16>(hb).x;
                        *reinterpret_cast<uint16_t*>(p0 + tc_off(r + kTcRows, t >> 3, 2 * kTcRows) + (t & 7) * 2) =
                            (uint16_t)(pack2<kBf16>(e - hi, 0.f) & 0xFFFFu);
                    }
                }
                // the previous product is finished before O^T is rescaled or
                // this tile's P^T released
                const bool pv_ok = n > 0 ? wait_pv(n) : true;
                if ((failed = tc_group_or(!pv_ok))) break;
                if (grow && !w.first()) {
                    float a[32];
#pragma unroll
                    for (int r = 0; r < 32; ++r) a[r] = __shfl_sync(kFull, a_lane, r);
#pragma unroll 1
                    for (int part = 0; part < kParts; ++part) {
                        float o[32];
                        tc_ld32(tmem + lane_addr + 64 + 32 * part, o);
#pragma unroll
                        for (int r = 0; r < 32; ++r) o[r] *= a[r];
                        tc_st32(tmem + lane_addr + 64 + 32 * part, o);
                    }
                    tc_wait_st();
                }
                fence_async_smem();
                tc_before_sync();
                mbar_arrive(bar(kTbP + (n & 1)));
                if (w.last()) {
                    // the unit segment's partial (m, l, o) of every member row
                    const bool o_ok = wait_pv(n + 1);
                    if ((failed = tc_group_or(!o_ok))) break;
                    u.locate(p, c, w.s, w.j);
                    float o[32];
                    tc_ld32(tmem + lane_addr + 64, o);
                    if constexpr (kParts == 2) {
                        float o2[32];
                        tc_ld32(tmem + lane_addr + 96, o2);
#pragma unroll
                        for (int r = 0; r < 32; ++r) o[r] += o2[r];
                    }
                    const bool split = (w.seg_i0 != 0) || (w.i != w.nt - 1);
                    const int64_t unit = (int64_t)w.s * ln.units + w.j;
                    float* o_rows;
                    float2* ml_rows;
                    if (split) {
                        const int64_t seg = (int64_t)blockIdx.x + unit;
                        o_rows = p.ws_o + seg * kTcRows * kTcD;
                        ml_rows = p.ws_ml + seg * kTcRows;
                    } else {
                        const int64_t row0 = ((int64_t)w.s * p.num_kv_heads + u.kh) * c.rows + kTcRows * u.rc;
                        o_rows = c.pre_o + row0 * kTcD;
                        ml_rows = c.pre_ml + row0;
                    }
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        if (r < u.nrows) o_rows[r * kTcD + t] = o[r];
                    float ls[32];
#pragma unroll
                    for (int r = 0; r < 32; ++r) ls[r] = l[r];
                    lred[warp][lane] = warp_reduce_scatter32<false>(ls);
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    if (warp == 0 && lane < u.nrows)
                        ml_rows[lane] = make_float2(m_lane, lred[0][lane] + lred[1][lane] + lred[2][lane] + lred[3][lane]);
                    asm volatile("bar.sync 1, 128;" ::: "memory");  // lred is free again
                }
                w.advance(ln);
            }
            if (failed) *abort = 1;
        }
    }
    // every role done (or left): free the tensor memory
    tc_before_sync();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc_after_sync();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
    }
    if (tid == 0 && abort_flag) raise_error(p.err, PKV_DEVERR_TIMEOUT);
}

}  // namespace pkv
