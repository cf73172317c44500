// paged_attention.cuh -- persistent, warp-specialised decode attention over a
// paged KV cache (sm_100a).
//
// What it computes: "PagedAttention不够用了之后" (thinkmoon.cn), section
// "PagedAttention 的计算优化": per sequence, gather the blocks named by the
// block table, softmax(q.K^T * scale) . V -- restricted to the sequence's
// logical length -- with the block-wise softmax of zwxr.cn section 3.3
// (running max m and normaliser l per block, merged by rescaling).
//
// How (B200 design):
//   * Work = tiles of 16 tokens of one (sequence, kv head, <= 8 q heads)
//     "unit".  All tiles of all units form one sequence of W tiles; CTA b of
//     the persistent grid takes the contiguous range [b*ceil(W/G), ...), so
//     every SM streams the same number of bytes whatever the length mix.
//     A unit cut by a range boundary leaves per-CTA partials (m, l, o) in the
//     workspace that pkv_merge_kernel combines exactly.
//   * Warp 8 (producer) translates each tile through the block table and
//     issues TMA box loads of its K and V rows (16 tokens x head_dim, one kv
//     head, 128-byte-swizzled) into a ring of shared-memory stages guarded by
//     mbarriers; the q rows of each unit arrive by a 1-D bulk copy together
//     with a small unit header.
//   * Warps 0..7 (consumers) take the tiles of a unit round-robin.  q.K^T and
//     P.V run on mma.sync tensor cores (tokens x heads and head_dim x heads
//     tiles, fp32 accumulators in registers) so one K/V read serves all q
//     heads of the GQA group; the online softmax runs on the accumulators.
//     FP8 E4M3 rows are converted to f16 in registers (exact).  fp32 caches
//     use CUDA cores.  At the end of a unit the warps' partial states are
//     merged through shared memory.
// Every wait is bounded; a wait that gives up raises PKV_DEVERR_TIMEOUT and
// all warps unwind together.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "pkv_device.cuh"

namespace pkv {

constexpr int kTileTokens = 16;   // tokens per pipeline tile
constexpr int kHeadsPerUnit = 8;  // q heads served by one KV read (one mma N tile)
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kSubBytes = kTileTokens * 128;  // one 128-byte-wide TMA box of 16 rows

struct DecodeParams {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const float* k_scale;  // device scalars (FP8 caches) or null
    const float* v_scale;
    float* ws_o;           // [(G + units) * hpu * D] partial outputs (unnormalised)
    float2* ws_ml;         // [(G + units) * hpu] partial (m, l), log2 domain
    int* err;
    int num_seqs, num_heads, num_kv_heads;
    int g;                 // q heads per kv head
    int nch;               // head chunks per kv head = ceil(g / 8)
    int hpu;               // heads per unit stride in the workspace = min(8, g)
    int max_blocks_per_seq, block_size, num_blocks;
    float scale_log2;      // scale * log2(e)
};

struct UnitHeader {
    int s, kh, c, nh;  // sequence, kv head, head chunk, real heads in the chunk
    int L;             // sequence length (clamped to the table capacity)
    int i0, i1;        // this CTA's tile range of the unit
    int split;         // 1: partial result goes to the workspace
    int seg;           // workspace segment of the partial
    int done;          // 1: no more units for this CTA
    int pad[6];
};
static_assert(sizeof(UnitHeader) == 64, "header size");

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }
__device__ __forceinline__ int ntiles_of(int L) { return (L + kTileTokens - 1) / kTileTokens; }

// Warp-collective: total tiles W = units_per_seq * sum_s ceil(L_s / 16);
// *bad_len is set when some length is negative or overruns its table row.
__device__ inline int64_t total_tiles(const int32_t* seq_lens, int S, int units, int cap,
                               bool* bad_len = nullptr) {
    const int lane = threadIdx.x & 31;
    int64_t tot = 0;
    bool bad = false;
    for (int s0 = 0; s0 < S; s0 += 256) {
        int part = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int s = s0 + lane * 8 + k;
            if (s < S) {
                const int L = __ldg(seq_lens + s);
                bad |= (L < 0 || L > cap);
                part += ntiles_of(clamp_len(L, cap));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(kFull, part, o);
        tot += part;
    }
    if (bad_len) *bad_len = __any_sync(kFull, bad);
    return tot * units;
}

struct SeqHit {
    int s;          // sequence holding tile P (num_seqs if none)
    int64_t base;   // index of its first tile
    int L;          // its clamped length
};

// Warp-collective: the sequence whose tiles contain global tile P.
__device__ inline SeqHit find_seq(const int32_t* seq_lens, int S, int units, int cap, int64_t P) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    for (int s0 = 0; s0 < S; s0 += 256) {
        int64_t w[8];
        int64_t part = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int s = s0 + lane * 8 + k;
            w[k] = (s < S) ? (int64_t)ntiles_of(clamp_len(__ldg(seq_lens + s), cap)) * units : 0;
            part += w[k];
        }
        int64_t incl = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(kFull, base + incl > P);
        if (hit) {
            const int src = __ffs(hit) - 1;
            int found = 0;
            int64_t at = 0;
            if (lane == src) {
                int64_t acc = base + incl - part;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (!found && acc + w[k] > P) { found = s0 + lane * 8 + k + 1; at = acc; }
                    acc += w[k];
                }
            }
            found = __shfl_sync(kFull, found, src) - 1;
            at = __shfl_sync(kFull, at, src);
            return SeqHit{found, at, clamp_len(__ldg(seq_lens + found), cap)};
        }
        base += __shfl_sync(kFull, incl, 31);
    }
    return SeqHit{S, base, 0};
}

// ----------------------------------------------------------------------------
// Per-variant traits and consumer math.
// ----------------------------------------------------------------------------
enum class Path { kMma16, kFp8, kF32 };

template <typename KvT, typename QT, int D_, Path P_>
struct Cfg {
    using kv_t = KvT;
    using q_t = QT;
    static constexpr Path kPath = P_;
    static constexpr int D = D_;
    static constexpr int kKvBytes = (int)sizeof(KvT);
    static constexpr int kQBytes = (int)sizeof(QT);
    static constexpr int kRowBytes = D * kKvBytes;
    static constexpr int kNSub = kRowBytes / 128;       // 128-byte TMA boxes per row
    static constexpr int kBoxElems = 128 / kKvBytes;    // elements per box row
    static constexpr int kTensorTile = kNSub * kSubBytes;
    static constexpr int kStageBytes = 2 * kTensorTile; // K tile + V tile
    static constexpr int kStages = (128 * 1024) / kStageBytes;
    static constexpr int kQData = kHeadsPerUnit * D * kQBytes;
    static constexpr int kQSlot = 128 + kQData;         // header (64 B) + pad + q rows
    static constexpr int kScrStride = D + 4;            // padded head stride (floats)
    static constexpr int kScrAcc = kConsumerWarps * kHeadsPerUnit * kScrStride * 4;
    static constexpr int kScrMl = kConsumerWarps * kHeadsPerUnit * 8;
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kOffStages + kStages * kStageBytes;
    static constexpr int kOffScr = kOffQ + 2 * kQSlot;
    static constexpr int kOffMl = kOffScr + kScrAcc;
    static constexpr int kOffBar = kOffMl + kScrMl;
    static constexpr int kNumBars = 2 * kStages + 4;
    static constexpr int kOffAbort = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffAbort + 16 + 1024;  // + alignment slack
    static_assert(kRowBytes % 128 == 0, "rows must be whole 128-byte boxes");
    static_assert(kStageBytes % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Zero rows [valid, 16) of a K or V tile (NSUB boxes of 16 x 128 B).  Used on
// a sequence's last tile so the unused slots (never written, any bits) cannot
// reach the tensor-core P.V product.
template <int kNSub>
__device__ __forceinline__ void zero_tail_rows(uint8_t* tile, int valid, int lane) {
    const int rows = kTileTokens - valid;
    const int per_sub = rows * 8;  // 16-byte chunks
    for (int idx = lane; idx < kNSub * per_sub; idx += 32) {
        const int sub = idx / per_sub, rem = idx % per_sub;
        const int row = valid + rem / 8, ch = rem % 8;
        *reinterpret_cast<uint4*>(tile + sub * kSubBytes + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
}

// Swizzled byte offset of 16-byte chunk `c` (of the whole row) in row t.
__device__ __forceinline__ uint32_t sw_off(int t, int c) {
    return (uint32_t)((c >> 3) * kSubBytes + t * 128 + ((((c & 7) ^ t) & 7) << 4));
}

// ---- 16-bit caches (f16 / bf16) and FP8 caches: tensor-core consumer --------
template <class C>
struct MmaConsumer {
    static constexpr bool kFp8 = C::kPath == Path::kFp8;
    static constexpr bool kOpBf16 = std::is_same<typename C::kv_t, __nv_bfloat16>::value;
    static constexpr int D = C::D;
    static constexpr int KS = D / 16;  // k-steps of q.K^T
    static constexpr int MT = D / 16;  // head_dim tiles of P.V

    uint32_t qf[KS][2];  // B fragments of q^T (heads = gid)
    float acc[MT][4];    // O^T fragments
    float m0, m1, l0, l1;
    float sl0, sl1;      // per-head score multipliers (log2 domain)

    __device__ void reset() {
#pragma unroll
        for (int i = 0; i < MT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    // q rows of the unit from shared memory; heads >= nh are zero.
    __device__ void load_q(const uint8_t* qs, int nh, float scale_log2, float kscale) {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        if constexpr (!kFp8) {
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qs);
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const bool on = gid < nh;
                qf[kk][0] = on ? q32[(gid * D + 16 * kk + 2 * tig) / 2] : 0u;
                qf[kk][1] = on ? q32[(gid * D + 16 * kk + 2 * tig + 8) / 2] : 0u;
            }
            sl0 = sl1 = scale_log2;
        } else {
            // q is f16 or bf16; K is converted to f16, so q goes to f16 too,
            // pre-scaled by a power of two per head (exact) to stay in range.
            // Thread (gid, tig) holds d = 32*tig + 4*kk + {0,1,2,3}: the same
            // permutation of the contraction index as its K fragments.
            using QT = typename C::q_t;
            const QT* qh = reinterpret_cast<const QT*>(qs) + gid * D + 32 * tig;
            float v[32];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                v[i] = (gid < nh) ? static_cast<float>(qh[i]) : 0.f;
                amax = fmaxf(amax, fabsf(v[i]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, 2));
            int e = 0;
            if (amax > 0.f && isfinite(amax)) frexpf(amax, &e);  // amax in [2^(e-1), 2^e)
            const float down = ldexpf(1.f, -e), up = ldexpf(1.f, e);
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                qf[kk][0] = pack2<false>(v[4 * kk] * down, v[4 * kk + 1] * down);
                qf[kk][1] = pack2<false>(v[4 * kk + 2] * down, v[4 * kk + 3] * down);
            }
            const float mine = up * kscale * scale_log2;  // multiplier of head gid
            sl0 = __shfl_sync(kFull, mine, (2 * tig) * 4);
            sl1 = __shfl_sync(kFull, mine, (2 * tig + 1) * 4);
        }
    }

    __device__ void tile(uint8_t* kt, uint8_t* vt, int valid) {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        if (valid < kTileTokens) zero_tail_rows<C::kNSub>(vt, valid, lane);
        const uint32_t kb = smem_u32(kt), vb = smem_u32(vt);
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (!kFp8) {
            const int r = lane & 7, mtx = lane >> 3;
            const int t = r + ((mtx & 1) << 3);
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a[4];
                ldsm_x4(a, kb + sw_off(t, 2 * kk + (mtx >> 1)));
                if (kk & 1) mma16816<kOpBf16>(sb, a, qf[kk][0], qf[kk][1]);
                else        mma16816<kOpBf16>(sa, a, qf[kk][0], qf[kk][1]);
            }
        } else {
            // K rows gid and gid+8, bytes [32*tig, 32*tig+32): two chunks each.
            uint4 r0a = *reinterpret_cast<const uint4*>(kt + sw_off(gid, 2 * tig));
            uint4 r0b = *reinterpret_cast<const uint4*>(kt + sw_off(gid, 2 * tig + 1));
            uint4 r1a = *reinterpret_cast<const uint4*>(kt + sw_off(gid + 8, 2 * tig));
            uint4 r1b = *reinterpret_cast<const uint4*>(kt + sw_off(gid + 8, 2 * tig + 1));
            const uint32_t w0[8] = {r0a.x, r0a.y, r0a.z, r0a.w, r0b.x, r0b.y, r0b.z, r0b.w};
            const uint32_t w1[8] = {r1a.x, r1a.y, r1a.z, r1a.w, r1b.x, r1b.y, r1b.z, r1b.w};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2((uint16_t)(w0[kk] & 0xffffu));
                a[1] = e4m3x2_to_f16x2((uint16_t)(w1[kk] & 0xffffu));
                a[2] = e4m3x2_to_f16x2((uint16_t)(w0[kk] >> 16));
                a[3] = e4m3x2_to_f16x2((uint16_t)(w1[kk] >> 16));
                if (kk & 1) mma16816<false>(sb, a, qf[kk][0], qf[kk][1]);
                else        mma16816<false>(sa, a, qf[kk][0], qf[kk][1]);
            }
        }
        // scores S^T[token][head]: (gid, 2tig), (gid, 2tig+1), (gid+8, 2tig), (gid+8, 2tig+1)
        float x0 = (sa[0] + sb[0]) * sl0, x1 = (sa[1] + sb[1]) * sl1;
        float x2 = (sa[2] + sb[2]) * sl0, x3 = (sa[3] + sb[3]) * sl1;
        if (gid >= valid) x0 = x1 = -INFINITY;
        if (gid + 8 >= valid) x2 = x3 = -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        constexpr bool kPBf16 = kOpBf16;  // P uses the operand type of the V product
        const uint32_t X0 = pack2<kPBf16>(ex2(x0 - mn0), ex2(x1 - mn1));
        const uint32_t X1 = pack2<kPBf16>(ex2(x2 - mn0), ex2(x3 - mn1));
        const float2 p0 = unpack2<kPBf16>(X0), p1 = unpack2<kPBf16>(X1);
        l0 = l0 * al0 + p0.x + p1.x;  // normaliser from the rounded P actually used
        l1 = l1 * al1 + p0.y + p1.y;
        const uint32_t b0 = movm_trans(X0), b1 = movm_trans(X1);  // P^T as mma B
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
            acc[mi][0] *= al0; acc[mi][1] *= al1; acc[mi][2] *= al0; acc[mi][3] *= al1;
        }
        if constexpr (!kFp8) {
            const int r = lane & 7, mtx = lane >> 3;
            const int t = r + ((mtx >> 1) << 3);
#pragma unroll
            for (int mi = 0; mi < MT; ++mi) {
                uint32_t a[4];
                ldsm_x4_trans(a, vb + sw_off(t, 2 * mi + (mtx & 1)));
                mma16816<kOpBf16>(acc[mi], a, b0, b1);
            }
        } else {
            // V^T fragments: thread gid owns d in [16*gid, 16*gid+16) (one chunk),
            // rows t = 2tig, 2tig+1, 2tig+8, 2tig+9; m-tile mi covers
            // d = 16*gid + 2*mi (row gid) and 16*gid + 2*mi + 1 (row gid+8).
            const uint4 R0 = *reinterpret_cast<const uint4*>(vt + sw_off(2 * tig, gid));
            const uint4 R1 = *reinterpret_cast<const uint4*>(vt + sw_off(2 * tig + 1, gid));
            const uint4 R8 = *reinterpret_cast<const uint4*>(vt + sw_off(2 * tig + 8, gid));
            const uint4 R9 = *reinterpret_cast<const uint4*>(vt + sw_off(2 * tig + 9, gid));
            const uint32_t q0[4] = {R0.x, R0.y, R0.z, R0.w}, q1[4] = {R1.x, R1.y, R1.z, R1.w};
            const uint32_t q8[4] = {R8.x, R8.y, R8.z, R8.w}, q9[4] = {R9.x, R9.y, R9.z, R9.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t X = prmt(q0[w], q1[w], 0x5140), Y = prmt(q0[w], q1[w], 0x7362);
                const uint32_t X8 = prmt(q8[w], q9[w], 0x5140), Y8 = prmt(q8[w], q9[w], 0x7362);
                uint32_t a[4];
                a[0] = e4m3x2_to_f16x2((uint16_t)(X & 0xffffu));
                a[1] = e4m3x2_to_f16x2((uint16_t)(X >> 16));
                a[2] = e4m3x2_to_f16x2((uint16_t)(X8 & 0xffffu));
                a[3] = e4m3x2_to_f16x2((uint16_t)(X8 >> 16));
                mma16816<false>(acc[2 * w], a, b0, b1);
                a[0] = e4m3x2_to_f16x2((uint16_t)(Y & 0xffffu));
                a[1] = e4m3x2_to_f16x2((uint16_t)(Y >> 16));
                a[2] = e4m3x2_to_f16x2((uint16_t)(Y8 & 0xffffu));
                a[3] = e4m3x2_to_f16x2((uint16_t)(Y8 >> 16));
                mma16816<false>(acc[2 * w + 1], a, b0, b1);
            }
        }
    }

    // Warp partial -> shared scratch: acc[w][head][d], ml[w][head].
    __device__ void store(float* scr, float2* ml, int warp) {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        float a0 = l0, a1 = l1;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            a0 += __shfl_xor_sync(kFull, a0, o);
            a1 += __shfl_xor_sync(kFull, a1, o);
        }
        float* s0 = scr + (warp * kHeadsPerUnit + 2 * tig) * C::kScrStride;
        float* s1 = s0 + C::kScrStride;
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
            int d0, d1;
            if constexpr (!kFp8) { d0 = 16 * mi + gid; d1 = d0 + 8; }
            else { d0 = 16 * gid + 2 * mi; d1 = d0 + 1; }
            s0[d0] = acc[mi][0]; s1[d0] = acc[mi][1];
            s0[d1] = acc[mi][2]; s1[d1] = acc[mi][3];
        }
        if (gid == 0) {
            ml[warp * kHeadsPerUnit + 2 * tig] = make_float2(m0, a0);
            ml[warp * kHeadsPerUnit + 2 * tig + 1] = make_float2(m1, a1);
        }
    }
};

// ---- fp32 caches: CUDA-core consumer ----------------------------------------
template <class C>
struct F32Consumer {
    static constexpr int D = C::D;
    static constexpr int CPR = D / 4;        // 16-byte chunks per row
    static constexpr int RPW = 32 / CPR;     // rows per warp-wide load (2 or 1)
    static constexpr int NIT = kTileTokens / RPW;
    float4 qv[kHeadsPerUnit];
    float4 acc[kHeadsPerUnit];
    float m[kHeadsPerUnit], l[kHeadsPerUnit];
    int nh;
    float sl;

    __device__ void reset() {
#pragma unroll
        for (int h = 0; h < kHeadsPerUnit; ++h) {
            acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
            m[h] = -INFINITY;
            l[h] = 0.f;
        }
    }
    __device__ void load_q(const uint8_t* qs, int nh_, float scale_log2, float) {
        const int lane = threadIdx.x & 31, c = lane % CPR;
        nh = nh_;
        sl = scale_log2;
        const float4* q4 = reinterpret_cast<const float4*>(qs);
#pragma unroll
        for (int h = 0; h < kHeadsPerUnit; ++h)
            qv[h] = (h < nh) ? q4[h * CPR + c] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __device__ void tile(uint8_t* kt, uint8_t* vt, int valid) {
        const int lane = threadIdx.x & 31, c = lane % CPR, rh = lane / CPR;
        float4 kr[NIT];
#pragma unroll
        for (int it = 0; it < NIT; ++it)
            kr[it] = *reinterpret_cast<const float4*>(kt + sw_off(it * RPW + rh, c));
        const int jt = (lane % CPR) >> 1;        // iteration whose full dot this lane ends with
        const int tok = jt * RPW + rh;
        float p[kHeadsPerUnit];
#pragma unroll
        for (int h = 0; h < kHeadsPerUnit; ++h) {
            if (h >= nh) { p[h] = 0.f; continue; }
            float v[NIT];
#pragma unroll
            for (int it = 0; it < NIT; ++it)
                v[it] = qv[h].x * kr[it].x + qv[h].y * kr[it].y + qv[h].z * kr[it].z + qv[h].w * kr[it].w;
            // halving butterfly over the CPR lanes of a row group
            int n = NIT;
#pragma unroll
            for (int msk = CPR / 2; msk >= 1; msk >>= 1) {
                if (n > 1) {
                    const bool up = (lane & msk) != 0;
                    const int half = n / 2;
#pragma unroll
                    for (int i = 0; i < NIT / 2; ++i) {
                        if (i < half) {
                            const float mine = up ? v[i + half] : v[i];
                            const float other = up ? v[i] : v[i + half];
                            v[i] = mine + __shfl_xor_sync(kFull, other, msk);
                        }
                    }
                    n = half;
                } else {
                    v[0] += __shfl_xor_sync(kFull, v[0], msk);
                }
            }
            float x = (tok < valid) ? v[0] * sl : -INFINITY;
            float mx = x;
#pragma unroll
            for (int o = 2; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
            const float mn = fmaxf(m[h], mx);
            const float al = ex2(m[h] - mn);
            m[h] = mn;
            p[h] = ex2(x - mn);
            l[h] = l[h] * al + ((lane & 1) ? 0.f : p[h]);
            acc[h].x *= al; acc[h].y *= al; acc[h].z *= al; acc[h].w *= al;
        }
#pragma unroll
        for (int it = 0; it < NIT; ++it) {
            const int t = it * RPW + rh;
            float4 vr = *reinterpret_cast<const float4*>(vt + sw_off(t, c));
            if (t >= valid) vr = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int h = 0; h < kHeadsPerUnit; ++h) {
                if (h >= nh) continue;
                const float pt = __shfl_sync(kFull, p[h], rh * CPR + 2 * it);
                acc[h].x += pt * vr.x; acc[h].y += pt * vr.y;
                acc[h].z += pt * vr.z; acc[h].w += pt * vr.w;
            }
        }
    }
    __device__ void store(float* scr, float2* ml, int warp) {
        const int lane = threadIdx.x & 31, c = lane % CPR, rh = lane / CPR;
#pragma unroll
        for (int h = 0; h < kHeadsPerUnit; ++h) {
            float4 a = acc[h];
            float ls = l[h];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) ls += __shfl_xor_sync(kFull, ls, o);
            if (RPW == 2) {
                a.x += __shfl_xor_sync(kFull, a.x, 16); a.y += __shfl_xor_sync(kFull, a.y, 16);
                a.z += __shfl_xor_sync(kFull, a.z, 16); a.w += __shfl_xor_sync(kFull, a.w, 16);
            }
            if (rh == 0)
                *reinterpret_cast<float4*>(scr + (warp * kHeadsPerUnit + h) * C::kScrStride + 4 * c) = a;
            if (lane == 0) ml[warp * kHeadsPerUnit + h] = make_float2(m[h], ls);
        }
    }
};

template <class C>
using ConsumerOf = typename std::conditional<C::kPath == Path::kF32, F32Consumer<C>, MmaConsumer<C>>::type;

// ----------------------------------------------------------------------------
// The kernel.
// ----------------------------------------------------------------------------
template <class C>
__global__ void __launch_bounds__(kThreads, 1)
pkv_decode_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem + C::kOffStages;
    uint8_t* qslots = smem + C::kOffQ;
    float* scr = reinterpret_cast<float*>(smem + C::kOffScr);
    float2* scr_ml = reinterpret_cast<float2*>(smem + C::kOffMl);
    const uint32_t bar0 = smem_u32(smem + C::kOffBar);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffAbort);
    auto full_bar = [&](int i) { return bar0 + 8u * i; };
    auto empty_bar = [&](int i) { return bar0 + 8u * (C::kStages + i); };
    auto qfull_bar = [&](int i) { return bar0 + 8u * (2 * C::kStages + i); };
    auto qempty_bar = [&](int i) { return bar0 + 8u * (2 * C::kStages + 2 + i); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::kStages; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(qfull_bar(i), 1);
            mbar_init(qempty_bar(i), kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    const int units_per_seq = p.num_kv_heads * p.nch;
    const int cap = p.max_blocks_per_seq * p.block_size;

    if (warp == kConsumerWarps) {
        // ======================= producer warp =======================
        if (lane == 0) { prefetch_tensormap(&tmk); prefetch_tensormap(&tmv); }
        bool bad_len = false;
        const int64_t W = total_tiles(p.seq_lens, p.num_seqs, units_per_seq, cap, &bad_len);
        if (bad_len && blockIdx.x == 0 && lane == 0) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
        const int64_t chunk = (W + gridDim.x - 1) / gridDim.x;
        const int64_t tb = min(W, (int64_t)blockIdx.x * chunk), te = min(W, tb + chunk);
        const int tpb = p.block_size / kTileTokens;
        uint32_t n = 0;
        int k = 0;
        bool ok = true;
        if (tb < te) {
            SeqHit hit = find_seq(p.seq_lens, p.num_seqs, units_per_seq, cap, tb);
            int s = hit.s, L = hit.L, nt = ntiles_of(L);
            int64_t base = hit.base;
            int j = (int)((tb - base) / nt);
            int i0 = (int)((tb - base) % nt);
            while (ok) {
                const int64_t T0 = base + (int64_t)j * nt;
                if (T0 >= te) break;
                const int i1 = (int)min((int64_t)nt, te - T0);
                const int kh = j / p.nch, c = j % p.nch;
                const int nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
                const int u = (s * p.num_kv_heads + kh) * p.nch + c;
                // ---- unit header + q rows
                const int slot = k & 1;
                ok = mbar_wait_bounded(qempty_bar(slot), ((k >> 1) & 1) ^ 1, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    UnitHeader* hd = reinterpret_cast<UnitHeader*>(qslots + slot * C::kQSlot);
                    hd->s = s; hd->kh = kh; hd->c = c; hd->nh = nh; hd->L = L;
                    hd->i0 = i0; hd->i1 = i1;
                    hd->split = (i0 != 0 || i1 != nt) ? 1 : 0;
                    hd->seg = (int)blockIdx.x + u;
                    hd->done = 0;
                    const uint32_t qbytes = (uint32_t)(nh * C::D * C::kQBytes);
                    const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q) +
                        ((int64_t)s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c) * C::D * C::kQBytes;
                    mbar_arrive_expect_tx(qfull_bar(slot), qbytes);
                    bulk_load(smem_u32(qslots + slot * C::kQSlot + 128), qsrc, qbytes, qfull_bar(slot));
                }
                ++k;
                // ---- tiles
                const int32_t* trow = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
                const int nblk = (L + p.block_size - 1) / p.block_size;
                int cbase = -64, creg = 0;
                for (int i = i0; i < i1; ++i) {
                    const int b = i / tpb;
                    if (b - cbase >= 32) {
                        cbase = b;
                        creg = (b + lane < nblk) ? __ldg(trow + b + lane) : 0;
                    }
                    int phys = __shfl_sync(kFull, creg, b - cbase);
                    if (phys < 0 || phys >= p.num_blocks) {
                        if (lane == 0) raise_error(p.err, PKV_DEVERR_BLOCK_ID);
                        phys = 0;
                    }
                    const int tok0 = (i % tpb) * kTileTokens;
                    const int st = (int)(n % C::kStages);
                    ok = mbar_wait_bounded(empty_bar(st), ((n / C::kStages) & 1) ^ 1, abort_flag);
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* kt = stages + st * C::kStageBytes;
                        uint8_t* vt = kt + C::kTensorTile;
                        mbar_arrive_expect_tx(full_bar(st), C::kStageBytes);
#pragma unroll
                        for (int sub = 0; sub < C::kNSub; ++sub)
                            tma_load_4d(smem_u32(kt + sub * kSubBytes), &tmk, full_bar(st),
                                        sub * C::kBoxElems, kh, tok0, phys);
#pragma unroll
                        for (int sub = 0; sub < C::kNSub; ++sub)
                            tma_load_4d(smem_u32(vt + sub * kSubBytes), &tmv, full_bar(st),
                                        sub * C::kBoxElems, kh, tok0, phys);
                    }
                    ++n;
                }
                if (!ok) break;
                // ---- next unit
                i0 = 0;
                if (++j == units_per_seq) {
                    j = 0;
                    base += (int64_t)units_per_seq * nt;
                    do {
                        ++s;
                        if (s >= p.num_seqs) break;
                        L = clamp_len(__ldg(p.seq_lens + s), cap);
                        nt = ntiles_of(L);
                    } while (nt == 0);
                    if (s >= p.num_seqs) break;
                }
            }
        }
        if (ok) {
            const int slot = k & 1;
            ok = mbar_wait_bounded(qempty_bar(slot), ((k >> 1) & 1) ^ 1, abort_flag);
            if (ok && lane == 0) {
                reinterpret_cast<UnitHeader*>(qslots + slot * C::kQSlot)->done = 1;
                mbar_arrive(qfull_bar(slot));
            }
        }
        if (!ok && lane == 0) raise_error(p.err, PKV_DEVERR_TIMEOUT);
        return;
    }

    // ======================= consumer warps =======================
    ConsumerOf<C> cs;
    constexpr int kCT = kConsumerWarps * 32;
    const int ctid = threadIdx.x;
    const float kscale = (C::kPath == Path::kFp8 && p.k_scale) ? __ldg(p.k_scale) : 1.f;
    const float vscale = (C::kPath == Path::kFp8 && p.v_scale) ? __ldg(p.v_scale) : 1.f;
    uint32_t n0 = 0;
    for (int k = 0;; ++k) {
        const int slot = k & 1;
        const bool got = mbar_wait_bounded(qfull_bar(slot), (k >> 1) & 1, abort_flag);
        const UnitHeader* hd = reinterpret_cast<const UnitHeader*>(qslots + slot * C::kQSlot);
        const bool stop = bar_sync_or(1, kCT, !got || hd->done);
        if (stop) break;
        const UnitHeader h = *hd;
        cs.load_q(qslots + slot * C::kQSlot + 128, h.nh, p.scale_log2, kscale);
        cs.reset();
        __syncwarp();
        if (lane == 0) mbar_arrive(qempty_bar(slot));
        const int ntile = h.i1 - h.i0;
        bool bad = false;
        for (int jt = warp; jt < ntile; jt += kConsumerWarps) {
            const uint32_t n = n0 + (uint32_t)jt;
            const int st = (int)(n % C::kStages);
            if (!mbar_wait_bounded(full_bar(st), (n / C::kStages) & 1, abort_flag)) { bad = true; break; }
            uint8_t* kt = stages + st * C::kStageBytes;
            const int tokb = (h.i0 + jt) * kTileTokens;
            cs.tile(kt, kt + C::kTensorTile, min(kTileTokens, h.L - tokb));
            fence_proxy_async_smem();  // generic writes (tail zeroing) before TMA reuse
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(st));
        }
        n0 += (uint32_t)ntile;
        if (bar_sync_or(1, kCT, bad)) break;
        // ---- merge the warps' partial states
        cs.store(scr, scr_ml, warp);
        bar_sync(1, kCT);
        const int D = C::D;
        for (int idx = ctid; idx < h.nh * D; idx += kCT) {
            const int hh = idx / D, d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, scr_ml[w * kHeadsPerUnit + hh].x);
            float ls = 0.f, o = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float2 ml = scr_ml[w * kHeadsPerUnit + hh];
                const float f = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
                ls += ml.y * f;
                o += scr[(w * kHeadsPerUnit + hh) * C::kScrStride + d] * f;
            }
            o *= vscale;
            if (!h.split) {
                using QT = typename C::q_t;
                QT* out = reinterpret_cast<QT*>(p.out) +
                          ((int64_t)h.s * p.num_heads + (int64_t)h.kh * p.g + kHeadsPerUnit * h.c + hh) * D + d;
                *out = from_f32<QT>(ls > 0.f ? o / ls : 0.f);
            } else {
                p.ws_o[((int64_t)h.seg * p.hpu + hh) * D + d] = o;
                if (d == 0) p.ws_ml[(int64_t)h.seg * p.hpu + hh] = make_float2(M, ls);
            }
        }
        bar_sync(1, kCT);
    }
}

// ----------------------------------------------------------------------------
// Exact merge of split units (zwxr.cn 3.3: M = max m_p,
// out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p) and zero output for
// empty sequences.  CTA b >= 1 owns the unit cut by boundary b (if it is the
// unit's first interior boundary); CTA 0 zeroes empty sequences.
// ----------------------------------------------------------------------------
template <typename QT>
__global__ void __launch_bounds__(256)
pkv_merge_kernel(const DecodeParams p, int D) {
    __shared__ int sh[8];
    const int units_per_seq = p.num_kv_heads * p.nch;
    const int cap = p.max_blocks_per_seq * p.block_size;
    const int G = gridDim.x;
    if (blockIdx.x == 0) {
        // rare: a thread per empty sequence writes its zero rows
        for (int s = threadIdx.x; s < p.num_seqs; s += blockDim.x) {
            if (clamp_len(__ldg(p.seq_lens + s), cap) != 0) continue;
            QT* out = reinterpret_cast<QT*>(p.out) + (int64_t)s * p.num_heads * D;
            for (int i = 0; i < p.num_heads * D; ++i) out[i] = from_f32<QT>(0.f);
        }
        return;
    }
    if (threadIdx.x < 32) {
        int flag = 0, s = 0, j = 0, bf = 0, bl = 0;
        const int64_t W = total_tiles(p.seq_lens, p.num_seqs, units_per_seq, cap);
        const int64_t chunk = (W + G - 1) / G;
        const int64_t P = (int64_t)blockIdx.x * chunk;
        if (P < W) {
            const SeqHit hit = find_seq(p.seq_lens, p.num_seqs, units_per_seq, cap, P);
            const int nt = ntiles_of(hit.L);
            j = (int)((P - hit.base) / nt);
            const int off = (int)((P - hit.base) % nt);
            const int64_t T0 = hit.base + (int64_t)j * nt;
            if (off != 0 && (int64_t)(blockIdx.x - 1) * chunk <= T0) {
                flag = 1;
                s = hit.s;
                bf = (int)(T0 / chunk);
                bl = (int)((T0 + nt - 1) / chunk);
            }
        }
        if (threadIdx.x == 0) { sh[0] = flag; sh[1] = s; sh[2] = j; sh[3] = bf; sh[4] = bl; }
    }
    __syncthreads();
    if (!sh[0]) return;
    const int s = sh[1], j = sh[2], bf = sh[3], bl = sh[4];
    const int kh = j / p.nch, c = j % p.nch;
    const int nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
    const int u = (s * p.num_kv_heads + kh) * p.nch + c;
    for (int idx = threadIdx.x; idx < nh * D; idx += blockDim.x) {
        const int hh = idx / D, d = idx % D;
        float M = -INFINITY;
        for (int b = bf; b <= bl; ++b) M = fmaxf(M, p.ws_ml[(int64_t)(b + u) * p.hpu + hh].x);
        float ls = 0.f, o = 0.f;
        for (int b = bf; b <= bl; ++b) {
            const float2 ml = p.ws_ml[(int64_t)(b + u) * p.hpu + hh];
            const float f = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
            ls += ml.y * f;
            o += p.ws_o[((int64_t)(b + u) * p.hpu + hh) * D + d] * f;
        }
        QT* out = reinterpret_cast<QT*>(p.out) +
                  ((int64_t)s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c + hh) * D + d;
        *out = from_f32<QT>(ls > 0.f ? o / ls : 0.f);
    }
}

}  // namespace pkv
