// cascade.cuh -- decode attention for sequences that share a prompt prefix
// (copy-on-write sharing, zwxr.cn section 3.4; ttlab.hopto.org section 2
// "共享区块"): the shared prefix blocks are streamed once per (group, kv head)
// and serve the query rows of every member of the group, instead of once per
// member.  The result is the same attention as pkv_paged_attention_decode:
// the prefix part and each member's own suffix are two partial softmaxes
// merged exactly with the block-wise (m, l) rule of zwxr.cn section 3.3.
//
// Passes (all on the caller's stream):
//   1. pkv_cascade_setup_kernel: per group, the effective shared prefix =
//      the longest run of leading blocks that every member's table shares,
//      capped by the requested prefix and by every member's length, in whole
//      blocks; scatter it to the members as their suffix start.
//   2. pkv_prefix_kernel: work unit = (group, kv head, chunk of 8*NT member
//      query rows); the same warp-level cp.async streaming as the decode
//      kernel, with NT tensor-core N tiles so one K/V tile feeds every member
//      row.  Whole units write their partial rows; split units leave
//      segments that pass 4 merges.
//   3. pkv_decode_kernel with seq_start = the suffix starts and partial
//      output for members (the ordinary path for everyone else).
//   4. pkv_cascade_combine_kernel: out = merge(prefix partial or segments,
//      suffix partial).
#pragma once

#include "paged_attention.cuh"

namespace pkv {

// Shortest prefix shared through the prefix pass, in 16-token tiles (the
// prefix kernel's query slots rely on it; shorter prefixes are decoded as
// part of each member's own sequence).
constexpr int kPrefixMinTiles = 2;

struct CascadeParams {
    const int32_t* grp_offsets;  // [G + 1] CSR offsets into grp_members
    const int32_t* grp_members;  // member sequence ids
    const int32_t* grp_prefix;   // [G] requested shared prefix (tokens)
    int32_t* prefix_eff;         // [G] effective shared prefix (tokens), written by setup
    int32_t* seq_start;          // [S] suffix start per sequence, written by setup
    int4* member_info;           // [S] member slot k < grp_offsets[G]: (sequence, group, index in
                                 // the group, 1 if the group shares a prefix), written by setup
    float* pre_o;                // [G * Hkv * R * D] prefix partial o (unnormalised)
    float2* pre_ml;              // [G * Hkv * R] prefix partial (m, l), log2 domain
    float* suf_o;                // [S * Hq * D] suffix partial o of members
    float2* suf_ml;              // [S * Hq]
    const float* pre_seg_o;      // prefix pass's split segments: [segments * R * D]
    const float2* pre_seg_ml;    // [segments * R]
    int2* seq_grp;               // [S] (group, index in the group) of a sequence with a shared prefix
    int64_t suffix_workers;      // workers (warps) of the suffix pass's tile split
    int split_grid;              // > 0: the prefix and suffix passes side by side on this many SMs
                                 // (cascade_prefix_ctas; prefix_workers / suffix_workers unused)
    int64_t prefix_workers;      // workers of the prefix pass (its tile split): warps, or CTAs
    int prefix_tile;             // tokens per tile of the prefix pass: 16, or 128 (tensor-core pass)
    int num_groups;
    int rows;                    // R = max_group_size * g (member query rows per kv head)
    int row_chunks;              // ceil(R / (8 * NT))
};

// Zeroes seq_start (and the suffix pass's CTA ticket after it) ahead of the
// setup pass, which is its programmatic dependent and waits for it only
// before its own writes.
__global__ void __launch_bounds__(256) pkv_cascade_zero_kernel(int32_t* a, int n) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) a[i] = 0;
}

// Pass 1 (one CTA per group; a programmatic dependent of the kernel that
// zeroes seq_start, waited for only before the writes): the group's
// effective prefix, scattered to its members as their suffix start.
__global__ void __launch_bounds__(256)
pkv_cascade_setup_kernel(const DecodeParams p, const CascadeParams c) {
    // the prefix pass (a programmatic dependent launch) may be scheduled now;
    // it waits for this grid before reading anything it writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int s_min, s_diff, s_bad;
    const int g = blockIdx.x, tid = threadIdx.x;
    const int cap = p.max_blocks_per_seq * p.block_size;
    const int o0 = __ldg(c.grp_offsets + g), o1 = __ldg(c.grp_offsets + g + 1);
    if (tid == 0) { s_min = cap; s_diff = 0x7fffffff; s_bad = 0; }
    __syncthreads();
    int minlen = cap, bad = 0;
    for (int i = o0 + tid; i < o1; i += blockDim.x) {
        const int s = __ldg(c.grp_members + i);
        if (s < 0 || s >= p.num_seqs) bad = 1;
        else minlen = min(minlen, clamp_len(__ldg(p.seq_lens + s), cap));
    }
    if (minlen < cap) atomicMin(&s_min, minlen);
    if (bad) atomicOr(&s_bad, 1);
    __syncthreads();
    int pre = __ldg(c.grp_prefix + g);
    pre = pre < 0 ? 0 : pre;
    minlen = s_min;
    // a request past a member's end, a member id outside [0, num_seqs) or a
    // group larger than max_group_size (c.rows / g) is flagged; such a group
    // (and any single-member group) shares nothing
    const bool fits = (o1 - o0) * p.g <= c.rows;
    if (tid == 0 && (pre > minlen || s_bad || !fits)) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
    const bool share = o1 - o0 > 1 && fits && !s_bad;
    const int nblk = share ? min(pre, minlen) / p.block_size : 0;
    // longest common run of leading physical blocks: thread per block, the
    // members' entries loaded independently
    if (nblk > 0) {
        const int32_t* first = p.block_tables + (int64_t)__ldg(c.grp_members + o0) * p.max_blocks_per_seq;
        for (int b = tid; b < nblk; b += blockDim.x) {
            const int f = __ldg(first + b);
            bool miss = false;
#pragma unroll 8
            for (int i = o0 + 1; i < o1; ++i)
                miss |= __ldg(p.block_tables + (int64_t)__ldg(c.grp_members + i) * p.max_blocks_per_seq + b) != f;
            if (miss) { atomicMin(&s_diff, b); break; }
        }
    }
    __syncthreads();
    int eff = min(nblk, s_diff) * p.block_size;
    if (eff < kPrefixMinTiles * 16) eff = 0;  // too short to be worth a shared pass
    asm volatile("griddepcontrol.wait;" ::: "memory");  // seq_start zeroed
    if (tid == 0) c.prefix_eff[g] = eff;
    for (int i = o0 + tid; i < o1; i += blockDim.x) {
        const int s = __ldg(c.grp_members + i);
        if (eff > 0) {  // eff > 0: every member id is valid
            c.seq_start[s] = eff;
            c.seq_grp[s] = make_int2(g, i - o0);
        }
        if (i < p.num_seqs) c.member_info[i] = make_int4(s, g, i - o0, eff > 0);
    }
}

// ---- tile math with NT tensor-core N tiles of 8 member query rows ----------
template <class C, int NT>
struct MmaRowsConsumer {
    static constexpr bool kOpBf16 = std::is_same<typename C::kv_t, __nv_bfloat16>::value;
    static constexpr int D = C::D;
    static constexpr int KS = D / 16;
    static constexpr int MT = D / 16;
    static constexpr int R = 8 * NT;  // rows per unit
    static_assert(NT == 2 || NT == 4, "row tiles");
    static_assert(C::kPath == Path::kMma16 && C::kTT == 16, "16-bit caches, 16-token tiles");

    float acc[MT][NT][4];
    float m[NT][2], l[NT][2];
    uint32_t qb;  // shared address of the unit's q rows (swizzled, R rows)
    float sl;
    // this lane's swizzled ldmatrix offsets (k-step / head_dim tile mod 4) in a
    // K tile, a V tile and the q slot; fixed for the kernel
    uint32_t ko[4], vo[4], qo[4];

    __device__ void init_lane() {
        const int lane = threadIdx.x & 31;
        const int r = lane & 7, mtx = lane >> 3;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            ko[k4] = sw_off<16>(r + ((mtx & 1) << 3), 2 * k4 + (mtx >> 1));
            vo[k4] = sw_off<16>(r + ((mtx >> 1) << 3), 2 * k4 + (mtx & 1));
            qo[k4] = sw_off<R>(8 * (mtx >> 1) + r, 2 * k4 + (mtx & 1));
        }
    }

    __device__ void reset() {
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int n = 0; n < NT; ++n) acc[i][n][0] = acc[i][n][1] = acc[i][n][2] = acc[i][n][3] = 0.f;
#pragma unroll
        for (int n = 0; n < NT; ++n) m[n][0] = m[n][1] = -INFINITY, l[n][0] = l[n][1] = 0.f;
    }
    // rows >= nrows of the slot are zeroed (they hold no member)
    __device__ void load_q(uint8_t* qs, int nrows, float scale_log2) {
        const int lane = threadIdx.x & 31;
        for (int idx = lane; idx < (R - nrows) * (C::kRowBytes / 16); idx += 32) {
            const int r = nrows + idx / (C::kRowBytes / 16), ch = idx % (C::kRowBytes / 16);
            *reinterpret_cast<uint4*>(qs + sw_off<R>(r, ch)) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        qb = smem_u32(qs);
        sl = scale_log2;
    }

    __device__ void tile(uint8_t* kt, uint8_t* vt, int valid) {
        const int lane = threadIdx.x & 31, gid = lane >> 2;
        if (valid < 16) zero_tail_rows<C::kNSub, 16>(vt, valid, lane);
        const uint32_t kb = smem_u32(kt), vb = smem_u32(vt);
        const int r = lane & 7, mtx = lane >> 3;
        float s[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, kb + ko[kk & 3] + (kk >> 2) * 2048);
#pragma unroll
            for (int n2 = 0; n2 < NT / 2; ++n2) {
                uint32_t b[4];  // b0, b1 of n-tile 2*n2 and of 2*n2+1
                ldsm_x4(b, qb + qo[kk & 3] + (kk >> 2) * (R * 128) + n2 * 2048);
                mma16816<kOpBf16>(s[2 * n2], a, b[0], b[1]);
                mma16816<kOpBf16>(s[2 * n2 + 1], a, b[2], b[3]);
            }
        }
        uint32_t b0[NT], b1[NT], c0[NT], c1[NT];
        // Row maxima of the tile.  The reference maximum m of a row moves
        // only when the tile's maximum passes it by more than 2^kLazyLog2
        // (then every row of the warp is rescaled at once); otherwise P =
        // 2^(x - m) <= 2^kLazyLog2, exact in the hi + lo parts, and o and l
        // stay relative to the same m (the (m, l, o) partials and the merge
        // accept any reference).
        constexpr float kLazyLog2 = 8.f;
        float x[NT][4], mx[NT][2];
        bool grow = false;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            x[n][0] = s[n][0] * sl; x[n][1] = s[n][1] * sl; x[n][2] = s[n][2] * sl; x[n][3] = s[n][3] * sl;
            if (gid >= valid) x[n][0] = x[n][1] = -INFINITY;
            if (gid + 8 >= valid) x[n][2] = x[n][3] = -INFINITY;
            float mx0 = fmaxf(x[n][0], x[n][2]), mx1 = fmaxf(x[n][1], x[n][3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
            }
            mx[n][0] = mx0;
            mx[n][1] = mx1;
            grow |= mx0 > m[n][0] + kLazyLog2 || mx1 > m[n][1] + kLazyLog2;
        }
        if (__any_sync(kFull, grow)) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float mn0 = fmaxf(m[n][0], mx[n][0]), mn1 = fmaxf(m[n][1], mx[n][1]);
                const float al0 = ex2(m[n][0] - mn0), al1 = ex2(m[n][1] - mn1);
                m[n][0] = mn0;
                m[n][1] = mn1;
                l[n][0] *= al0;
                l[n][1] *= al1;
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    acc[mi][n][0] *= al0; acc[mi][n][1] *= al1;
                    acc[mi][n][2] *= al0; acc[mi][n][3] *= al1;
                }
            }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const float e0 = ex2(x[n][0] - m[n][0]), e1 = ex2(x[n][1] - m[n][1]);
            const float e2 = ex2(x[n][2] - m[n][0]), e3 = ex2(x[n][3] - m[n][1]);
            const uint32_t X0 = pack2<kOpBf16>(e0, e1), X1 = pack2<kOpBf16>(e2, e3);
            if constexpr (kOpBf16) {  // P as hi + lo bf16 parts (see MmaConsumer)
                const float2 h0 = unpack2<true>(X0), h1 = unpack2<true>(X1);
                c0[n] = movm_trans(pack2<true>(e0 - h0.x, e1 - h0.y));
                c1[n] = movm_trans(pack2<true>(e2 - h1.x, e3 - h1.y));
                l[n][0] += e0 + e2;
                l[n][1] += e1 + e3;
            } else {
                const float2 p0 = unpack2<false>(X0), p1 = unpack2<false>(X1);
                l[n][0] += p0.x + p1.x;
                l[n][1] += p0.y + p1.y;
                c0[n] = c1[n] = 0u;
            }
            b0[n] = movm_trans(X0);
            b1[n] = movm_trans(X1);
        }
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
            uint32_t a[4];
            ldsm_x4_trans(a, vb + vo[mi & 3] + (mi >> 2) * 2048);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                mma16816<kOpBf16>(acc[mi][n], a, b0[n], b1[n]);
                if constexpr (kOpBf16) mma16816<true>(acc[mi][n], a, c0[n], c1[n]);
            }
        }
    }

    // Partial (m, l, o) of every valid row: to the workspace segment (split
    // unit) or straight to the prefix partial rows.
    __device__ void finish(float* o_rows, float2* ml_rows, int nrows) {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            float a0 = l[n][0], a1 = l[n][1];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                a0 += __shfl_xor_sync(kFull, a0, o);
                a1 += __shfl_xor_sync(kFull, a1, o);
            }
            const int h0 = 8 * n + 2 * tig, h1 = h0 + 1;
#pragma unroll
            for (int mi = 0; mi < MT; ++mi) {
                const int d0 = 16 * mi + gid, d1 = d0 + 8;
                if (h0 < nrows) { o_rows[h0 * D + d0] = acc[mi][n][0]; o_rows[h0 * D + d1] = acc[mi][n][2]; }
                if (h1 < nrows) { o_rows[h1 * D + d0] = acc[mi][n][1]; o_rows[h1 * D + d1] = acc[mi][n][3]; }
            }
            if (gid == 0) {
                if (h0 < nrows) ml_rows[h0] = make_float2(m[n][0], a0);
                if (h1 < nrows) ml_rows[h1] = make_float2(m[n][1], a1);
            }
        }
    }
};

// Pass 2: the shared prefixes, every warp an independent worker over an equal
// share of all (group, kv head, row chunk) tiles.
template <class C, int NT>
__global__ void __launch_bounds__(C::kWarps * 32, 1)
pkv_prefix_kernel(const DecodeParams p, const CascadeParams c) {
    // launched as a programmatic dependent of the setup pass: its results
    // (prefix_eff, seq_start, member_info) are complete and visible only after
    // the wait; then the suffix pass may be scheduled (it reads seq_start)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int R = 8 * NT;
    constexpr int kQSlot = R * C::kRowBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // per warp: the K/V ring and two query slots used by alternate units.  A
    // slot is refilled while the issue walk, at most kStages-1 tiles ahead,
    // starts the unit after next; every unit but a worker's first holds at
    // least kPrefixMinTiles = kStages-1 tiles (setup shares no shorter
    // prefix), so the compute walk has left the slot's previous unit by then.
    static_assert(C::kStages - 1 <= kPrefixMinTiles, "query slots need units of kStages-1 tiles");
    uint8_t* stages = smem + warp * (C::kStages * C::kStageBytes + 2 * kQSlot);
    uint8_t* qslots = stages + C::kStages * C::kStageBytes;

    const Lens<false> ln{c.prefix_eff, nullptr, c.num_groups, p.num_kv_heads * c.row_chunks, 0x7fffffff};
    const int64_t workers = (int64_t)gridDim.x * C::kWarps;
    const int64_t wid = (int64_t)blockIdx.x * C::kWarps + warp;
    const int64_t W = total_tiles<16>(ln);
    const int64_t chunk = (W + workers - 1) / workers;
    const int64_t tb = min(W, wid * chunk), te = min(W, tb + chunk);
    if (tb >= te) return;

    // member rows of unit j of group g: rows [R*rc, R*rc + R) of the group's
    // members x q heads of kv head kh (row = member * g + head).  Looked up
    // once per unit: per tile, the loads would sit behind the previous
    // tile's copies (a compiler memory barrier) and stall the issue.
    struct UnitInfo {
        int s = -1, j = -1, kh, rc, nrows, o0, first_member;
    };
    auto unit_rows = [&](const Walk<16>& w, UnitInfo& u) {
        if (u.s == w.s && u.j == w.j) return;
        u.s = w.s;
        u.j = w.j;
        u.kh = w.j / c.row_chunks;
        u.rc = w.j % c.row_chunks;
        u.o0 = __ldg(c.grp_offsets + w.s);
        const int total = (__ldg(c.grp_offsets + w.s + 1) - u.o0) * p.g;
        u.nrows = max(0, min(R, total - R * u.rc));
        u.first_member = __ldg(c.grp_members + u.o0);
    };
    UnitInfo iu, cu;  // issue walk's and compute walk's units
    IssueLane<C> il;
    il.init(p);
    const int lg_bs = 31 - __clz(p.block_size);
    auto issue = [&](const Walk<16>& w, TablePrefetch& tp, uint8_t* stg, uint8_t* qslot) {
        unit_rows(w, iu);
        const int kh = iu.kh, rc = iu.rc, nrows = iu.nrows, o0 = iu.o0, first_member = iu.first_member;
        const int tok = w.i * 16;
        const int bmask = (1 << lg_bs) - 1;
        const int nblk = (w.L + bmask) >> lg_bs;
        int phys = tp.get(p, first_member, tok >> lg_bs, nblk, lane);
        if (phys < 0 || phys >= p.num_blocks) {
            if (lane == 0) raise_error(p.err, PKV_DEVERR_BLOCK_ID);
            phys = 0;
        }
        const int64_t base = ((((int64_t)phys << lg_bs) + (tok & bmask)) * p.num_kv_heads + kh) * C::kRowBytes;
        const uint32_t kdst = smem_u32(stg), vdst = smem_u32(stg + C::kTensorTile);
        const uint8_t* kl = p.key_cache + il.goff;
        const uint8_t* vl = p.value_cache + il.goff;
#pragma unroll
        for (int it = 0; it < 16 / C::kRowsPerInst; ++it) {
            const int64_t off = base + it * il.gstep;
            const uint32_t so = il.so[it % IssueLane<C>::kP] + (it / IssueLane<C>::kP) * 1024;
            cp_async16(kdst + so, kl + off);
            cp_async16(vdst + so, vl + off);
        }
        if (w.first()) {
            constexpr int CPR = C::kRowBytes / 16;
            for (int idx = lane; idx < nrows * CPR; idx += 32) {
                const int rr = idx / CPR, ch = idx % CPR;
                const int row = R * rc + rr;                      // member row within the group
                const int s = __ldg(c.grp_members + o0 + row / p.g);
                const uint8_t* src = reinterpret_cast<const uint8_t*>(p.q) +
                    ((int64_t)s * p.num_heads + (int64_t)kh * p.g + row % p.g) * C::kRowBytes + ch * 16;
                cp_async16(smem_u32(qslot + sw_off<R>(rr, ch)), src);
            }
        }
    };

    Walk<16> iw, cw;
    iw.init(ln, tb, te);
    cw = iw;
    TablePrefetch tp;
#pragma unroll 1
    for (int k = 0; k < C::kStages - 1; ++k) {
        if (!iw.done) issue(iw, tp, stages + k * C::kStageBytes, qslots + (iw.ord & 1) * kQSlot);
        cp_async_commit();
        iw.advance(ln);
    }
    MmaRowsConsumer<C, NT> cs;
    cs.init_lane();
#pragma unroll 1
    for (int n = 0; !cw.done; ++n) {
        if (!iw.done)
            issue(iw, tp, stages + ((n + C::kStages - 1) % C::kStages) * C::kStageBytes,
                  qslots + (iw.ord & 1) * kQSlot);
        cp_async_commit();
        iw.advance(ln);
        cp_async_wait<C::kStages - 1>();
        __syncwarp();
        unit_rows(cw, cu);
        const int kh = cu.kh, rc = cu.rc, nrows = cu.nrows;
        if (cw.first()) {
            cs.load_q(qslots + (cw.ord & 1) * kQSlot, nrows, p.scale_log2);
            cs.reset();
        }
        uint8_t* kt = stages + (n % C::kStages) * C::kStageBytes;
        cs.tile(kt, kt + C::kTensorTile, min(16, cw.L - cw.i * 16));
        if (cw.last()) {
            const bool split = (cw.seg_i0 != 0) || (cw.i != cw.nt - 1);
            const int64_t unit = (int64_t)cw.s * ln.units + cw.j;
            if (split) {
                const int64_t seg = wid + unit;
                cs.finish(p.ws_o + seg * R * C::D, p.ws_ml + seg * R, nrows);
            } else {
                const int64_t row0 = ((int64_t)cw.s * p.num_kv_heads + kh) * c.rows + R * rc;
                cs.finish(c.pre_o + row0 * C::D, c.pre_ml + row0, nrows);
            }
        }
        __syncwarp();
        cw.advance(ln);
    }
    cp_async_wait<0>();
}

// Sum over groups g' < g of the tiles (tt tokens each) of their units
// (warp-collective): the index of group g's first tile in the prefix pass's
// tile sequence (g = the number of groups: the total).
__device__ inline int64_t group_tile_base(const Lens<false>& ln, int g, int tt) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    for (int g0 = 0; g0 < g; g0 += 32) {
        const int gi = g0 + lane;
        int64_t t = gi < g ? (int64_t)((ln.eff(gi) + tt - 1) / tt) * ln.units : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
        base += t;
    }
    return base;
}

// Pass 4: out[s, h] = merge(prefix partial, suffix partial) for every member
// of a group with a shared prefix; one warp per (member, q head).  The
// prefix partial of the member's row is the prefix kernel's whole-unit row,
// or, for a unit split between workers, its segments merged here (folded
// four at a time with the suffix partial last, the (m, l) rule of zwxr.cn
// section 3.3).
template <typename QT, int D, int NT>
__global__ void __launch_bounds__(256)
pkv_cascade_combine_kernel(const DecodeParams p, const CascadeParams c) {
    // a programmatic dependent of the suffix pass's merge: every partial (the
    // prefix pass's included, which the suffix pass waited for) is complete
    // and visible after the wait; before it, only what the setup pass wrote
    // is read (complete before this grid starts: every pass between waited
    // for it before releasing its dependent)
    constexpr int R = 8 * NT;
    constexpr int PER = D / 32;
    const int k = blockIdx.x;  // member slot
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = (int)blockIdx.y * 8 + warp;
    const int total = __ldg(c.grp_offsets + c.num_groups);
    const int4 info = c.member_info[k];  // (s, g, index in group, shared)
    if (k >= total || !info.w || h >= p.num_heads) return;  // no sharing: the suffix pass wrote out
    const int s = info.x, g = info.y, mi = info.z;
    const int kh = h / p.g;
    const int row = mi * p.g + h % p.g;                     // member row of the group
    const int rc = row / R, rr = row % R;
    const Lens<false> ln{c.prefix_eff, nullptr, c.num_groups, p.num_kv_heads * c.row_chunks, 0x7fffffff};
    const int j = kh * c.row_chunks + rc;                   // unit of the group
    const int tt = c.prefix_tile;
    const int nt = (ln.eff(g) + tt - 1) / tt;
    const int64_t W = group_tile_base(ln, c.num_groups, tt);
    const int64_t chunk = (W + c.prefix_workers - 1) / c.prefix_workers;
    const int64_t T0 = group_tile_base(ln, g, tt) + (int64_t)j * nt;
    const int64_t bf = T0 / chunk, bl = (T0 + nt - 1) / chunk;
    const int64_t unit = (int64_t)g * ln.units + j;

    float M = -INFINITY, ls = 0.f, o[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;
    auto fold = [&](const float2 (&ml)[4], const float (&v)[4][PER]) {
        float Mb = M;
#pragma unroll
        for (int q = 0; q < 4; ++q) Mb = fmaxf(Mb, ml[q].x);
        if (Mb == -INFINITY) return;
        const float fo = M == -INFINITY ? 0.f : ex2(M - Mb);
        ls *= fo;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] *= fo;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float f = ml[q].x == -INFINITY ? 0.f : ex2(ml[q].x - Mb);
            ls += ml[q].y * f;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] += v[q][e] * f;
        }
        M = Mb;
    };
    // the prefix partial: one whole-unit row, or segments bf..bl; then the
    // suffix partial (index n of the sequence of partials)
    const int n = bf == bl ? 1 : (int)(bl - bf + 1);
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i0 = 0; i0 <= n; i0 += 4) {
        float2 ml[4];
        float v[4][PER];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = i0 + q;
            ml[q] = make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int e = 0; e < PER; ++e) v[q][e] = 0.f;
            const float* src = nullptr;
            if (i < n) {
                if (bf == bl) {
                    const int64_t pr = ((int64_t)g * p.num_kv_heads + kh) * c.rows + row;
                    ml[q] = c.pre_ml[pr];
                    src = c.pre_o + pr * D;
                } else {
                    const int64_t sg = (bf + i + unit) * R + rr;
                    ml[q] = c.pre_seg_ml[sg];
                    src = c.pre_seg_o + sg * D;
                }
            } else if (i == n) {
                const int64_t sr = (int64_t)s * p.num_heads + h;
                ml[q] = c.suf_ml[sr];
                src = c.suf_o + sr * D;
            }
            if (src) {
#pragma unroll
                for (int e = 0; e < PER; ++e) v[q][e] = src[lane + 32 * e];
            }
        }
        fold(ml, v);
    }
    QT* out = reinterpret_cast<QT*>(p.out) + ((int64_t)s * p.num_heads + h) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) out[lane + 32 * e] = from_f32<QT>(ls > 0.f ? o[e] / ls : 0.f);
}


// Pass 4 for batches whose length scan takes one round of a warp (the
// suffix pass then skips its merge kernel): one warp per (sequence s, q head
// h) folds, in order, the prefix partial of s's row (if s shares a prefix:
// the prefix kernel's whole-unit row or its split segments) and the suffix
// pass's partials of s's unit (its whole-unit partial, or the segments of
// the workers it was split between), with the (m, l) rule of zwxr.cn
// section 3.3, and writes out.  A sequence without a shared prefix whose
// unit was whole was written by the suffix pass itself; an empty one gets
// zeros.  Everything before the dependency wait reads only what the setup
// pass wrote, which is complete before this grid starts (every pass between
// waited for it before releasing its dependent).
template <typename QT, int D, int NT>
__global__ void __launch_bounds__(256)
pkv_cascade_finish_kernel(const DecodeParams p, const CascadeParams c) {
    constexpr int R = 8 * NT;
    constexpr int PER = D / 32;
    const int s = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int h = (int)blockIdx.y * 8 + warp;
    if (h >= p.num_heads) return;
    const int kh = h / p.g, hg = h % p.g;
    // the suffix pass's unit of (s, h): its tile range and the workers holding it
    const Lens<true> lsuf{p.seq_lens, c.seq_start, p.num_seqs, p.num_kv_heads * p.nch,
                          p.max_blocks_per_seq * p.block_size};
    int64_t Ws, base;
    seq_tile_base<kTileTokens>(lsuf, s, &Ws, &base);
    const int st = lsuf.first(s), eff = lsuf.eff(s);
    const int cch = hg / kHeadsPerUnit, hh = hg % kHeadsPerUnit;
    const int nts = ntiles_of<kTileTokens>(eff);
    const Lens<false> ln{c.prefix_eff, nullptr, c.num_groups, p.num_kv_heads * c.row_chunks, 0x7fffffff};
    const int tt = c.prefix_tile;
    const int64_t Wpre = group_tile_base(ln, c.num_groups, tt);
    // the two passes' worker counts (their tile splits)
    int64_t suffix_workers = c.suffix_workers, prefix_workers = c.prefix_workers;
    if (c.split_grid > 0) {
        const int P = cascade_prefix_ctas(Wpre, tt, Ws, kTileTokens, c.split_grid);
        prefix_workers = max(1, P);
        suffix_workers = (int64_t)(c.split_grid - P) * kWarps16;
    }
    const int64_t chunk_s = (Ws + suffix_workers - 1) / suffix_workers;
    const int64_t T0s = base + (int64_t)(kh * p.nch + cch) * nts;
    const int64_t us = ((int64_t)s * p.num_kv_heads + kh) * p.nch + cch;
    const int64_t sbf = eff > 0 ? T0s / chunk_s : 0, sbl = eff > 0 ? (T0s + nts - 1) / chunk_s : -1;
    const bool suf_whole = eff > 0 && sbf == sbl;
    if (st == 0 && suf_whole) return;  // written by the suffix pass
    const int nsuf = eff == 0 ? 0 : (suf_whole ? 1 : (int)(sbl - sbf + 1));
    // the prefix partial of the row (sequences with a shared prefix)
    int npre = 0;
    int64_t pr = 0, pbf = 0, punit = 0;
    int rr = 0;
    if (st > 0) {
        const int2 gm = c.seq_grp[s];
        const int g = gm.x, row = gm.y * p.g + hg;
        const int rc = row / R;
        rr = row % R;
        const int j = kh * c.row_chunks + rc;
        const int nt = (ln.eff(g) + tt - 1) / tt;
        const int64_t chunk = (Wpre + prefix_workers - 1) / prefix_workers;
        const int64_t T0 = group_tile_base(ln, g, tt) + (int64_t)j * nt;
        pbf = T0 / chunk;
        const int64_t pbl = (T0 + nt - 1) / chunk;
        punit = (int64_t)g * ln.units + j;
        pr = ((int64_t)g * p.num_kv_heads + kh) * c.rows + row;
        npre = pbf == pbl ? 1 : (int)(pbl - pbf + 1);
        if (pbf == pbl) pbf = -1;  // the whole-unit row
    }
    // the partials are complete and visible after the wait
    asm volatile("griddepcontrol.wait;" ::: "memory");

    float M = -INFINITY, ls = 0.f, o[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;
    const int n = npre + nsuf;
    for (int i0 = 0; i0 < n; i0 += 4) {
        float2 ml[4];
        float v[4][PER];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int i = i0 + q;
            ml[q] = make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int e = 0; e < PER; ++e) v[q][e] = 0.f;
            const float* src = nullptr;
            if (i < npre) {
                if (pbf < 0) {
                    ml[q] = c.pre_ml[pr];
                    src = c.pre_o + pr * D;
                } else {
                    const int64_t sg = (pbf + i + punit) * R + rr;
                    ml[q] = c.pre_seg_ml[sg];
                    src = c.pre_seg_o + sg * D;
                }
            } else if (i < n) {
                if (suf_whole) {
                    const int64_t sr = (int64_t)s * p.num_heads + h;
                    ml[q] = c.suf_ml[sr];
                    src = c.suf_o + sr * D;
                } else {
                    const int64_t sg = (sbf + (i - npre) + us) * p.hpu + hh;
                    ml[q] = p.ws_ml[sg];
                    src = p.ws_o + sg * D;
                }
            }
            if (src) {
#pragma unroll
                for (int e = 0; e < PER; ++e) v[q][e] = src[lane + 32 * e];
            }
        }
        float Mb = M;
#pragma unroll
        for (int q = 0; q < 4; ++q) Mb = fmaxf(Mb, ml[q].x);
        if (Mb == -INFINITY) continue;
        const float fo = M == -INFINITY ? 0.f : ex2(M - Mb);
        ls *= fo;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] *= fo;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float f = ml[q].x == -INFINITY ? 0.f : ex2(ml[q].x - Mb);
            ls += ml[q].y * f;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] += v[q][e] * f;
        }
        M = Mb;
    }
    QT* out = reinterpret_cast<QT*>(p.out) + ((int64_t)s * p.num_heads + h) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) out[lane + 32 * e] = from_f32<QT>(ls > 0.f ? o[e] / ls : 0.f);
}

}  // namespace pkv
