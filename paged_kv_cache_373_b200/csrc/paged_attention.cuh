// paged_attention.cuh -- decode attention over a paged KV cache (sm_100a).
//
// What it computes: "PagedAttention不够用了之后" (thinkmoon.cn), section
// "PagedAttention 的计算优化": per sequence, gather the blocks named by the
// block table and compute softmax(q.K^T * scale) . V over the sequence's
// logical length, using the block-wise softmax of zwxr.cn section 3.3
// (running max m and normaliser l, merged by rescaling).
//
// How (B200 design):
//   * Work unit = (sequence, kv head, <= 8 q heads of its GQA group); a unit
//     of length L is ceil(L/16) tiles of 16 tokens.  The tiles of all units
//     are laid end to end (W tiles) and every warp of the persistent grid is a
//     worker that takes one contiguous range of ceil(W / workers) tiles, so
//     every warp streams the same number of KV bytes whatever the length mix.
//   * A worker streams its tiles through its own ring of shared-memory
//     stages with 16-byte cp.async loads (the row gather of a paged cache is
//     ~50 % faster this way than with TMA boxes on B200: 6.9 vs 4.5 TB/s
//     measured for 256-byte rows), block-table entries prefetched 32 blocks
//     ahead, the q rows of each unit riding in the same async group.
//   * Tile math on tensor cores: S^T[16 tokens x 8 heads] = K q^T and
//     O^T[head_dim x 8 heads] += V^T P^T with mma.sync (fp32 accumulators in
//     registers) so one K/V read serves every q head of the group; the online
//     softmax runs on the accumulator fragments (exp2 domain, fp32).  FP8 E4M3
//     rows convert exactly to f16 in registers; fp32 caches use CUDA cores.
//   * A worker whose range holds a whole unit writes the output; a unit cut
//     by range boundaries leaves per-worker partials (m, l, o) that
//     pkv_merge_kernel combines exactly.
// No warp waits on another warp: the only synchronisation is each warp's own
// cp.async groups, so nothing in the kernel can wait forever.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "pkv_device.cuh"

namespace pkv {

constexpr int kTileTokens = 16;    // tokens per pipeline tile (32 for FP8 caches with 32-token blocks)
constexpr int kHeadsPerUnit = 8;   // q heads served by one KV read (one mma N tile)
constexpr int kMaxWarpsPerCta = 12; // workspace is sized for this many workers per CTA
constexpr int kWarps16 = 8;         // warps (workers) per CTA of the 16-bit-cache decode kernels
constexpr int kMaxCtas = 1 << 20;   // bound on num_ctas: every worker count (CTAs x warps) fits a grid dimension

struct DecodeParams {
    void* out;
    const void* q;
    const uint8_t* key_cache;
    const uint8_t* value_cache;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const float* k_scale;  // device scalars (FP8 caches) or null
    const float* v_scale;
    float* ws_o;           // [(workers + units) * hpu * D] partial outputs (unnormalised)
    float2* ws_ml;         // [(workers + units) * hpu] partial (m, l), log2 domain
    int* err;
    int num_seqs, num_heads, num_kv_heads;
    int g;                 // q heads per kv head
    int nch;               // head chunks per kv head = ceil(g / 8)
    int hpu;               // heads per unit stride in the workspace = min(8, g)
    int max_blocks_per_seq, block_size, num_blocks;
    float scale_log2;      // scale * log2(e)
};
// (DecodeParams is kept at 128 bytes: growing it changed the code generated
// for the decode kernel and cost 3-4% of its bandwidth.)

// Cascade suffix pass only (a second kernel argument, empty otherwise): the
// first token attended per sequence, and for sequences with a non-zero start
// the unnormalised o and (m, l) partials that replace out.
template <bool kSuffix> struct SuffixArg {
    static constexpr const int32_t* seq_start = nullptr;
};
template <> struct SuffixArg<true> {
    const int32_t* seq_start;  // [num_seqs]
    float* part_o;             // [num_seqs * num_heads * D]
    float2* part_ml;           // [num_seqs * num_heads]
    // The passes side by side (prefix_tile > 0): the grid's SMs are split
    // between the cascade's prefix pass and this one by cascade_prefix_ctas;
    // the CTAs past this pass's share leave at once.
    const int32_t* prefix_eff; // [num_groups] shared prefix per group
    int* cta_ticket;           // zeroed before the pass: its CTAs take worker slots in order of arrival
    int num_groups;
    int prefix_units;          // prefix units per group (kv heads x row chunks)
    int prefix_tile;           // tokens per prefix tile, 0: the passes run one after the other
};

// The cascade's prefix and suffix passes side by side on disjoint SMs: of a
// grid of `grid` SMs the prefix pass takes P (its CTAs [0, P)) and the
// suffix pass the other grid - P (its CTAs [0, grid - P)), in proportion to
// the time each needs: Wp tiles of tp tokens against Ws tiles of ts (the
// same K/V bytes per token), a prefix token weighted kPrefixCost /
// kSuffixCost (an SM of the prefix pass streamed ~31 GB/s beside the suffix
// pass, one of the suffix pass ~45 GB/s).  Integer arithmetic: every pass
// computes the same split from the same setup results.  With nothing shared
// the suffix pass takes the whole grid; otherwise each pass keeps at least
// one CTA.
constexpr int kPrefixCost = 3, kSuffixCost = 2;
__device__ __forceinline__ int cascade_prefix_ctas(int64_t Wp, int tp, int64_t Ws, int ts, int grid) {
    const int64_t bp = Wp * tp * kPrefixCost, bs = Ws * ts * kSuffixCost;
    if (bp == 0 || grid < 2) return 0;
    const int64_t P = (grid * bp + (bp + bs) / 2) / (bp + bs);
    return (int)min((int64_t)grid - 1, max((int64_t)1, P));
}

// Warp-collective: tiles of the prefix pass, units * sum_g ceil(eff_g / tp).
__device__ inline int64_t cascade_prefix_tiles(const int32_t* prefix_eff, int num_groups, int units, int tp) {
    const int lane = threadIdx.x & 31;
    int64_t t = 0;
    for (int g = lane; g < num_groups; g += 32) t += (__ldg(prefix_eff + g) + tp - 1) / tp;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(kFull, t, o);
    return t * units;
}

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// Per-sequence token ranges [start_s, L_s) the kernel attends over; kStart
// false: every range starts at token 0 (start is not read).
template <bool kStart>
struct Lens {
    static constexpr bool kHasStart = kStart;
    const int32_t* len;
    const int32_t* start;
    int S, units, cap;
    // raw seq_lens / start entries of sequence s (start 0 when kStart is false)
    __device__ __forceinline__ int raw_len(int s) const { return __ldg(len + s); }
    __device__ __forceinline__ int raw_start(int s) const {
        if constexpr (!kStart) return 0;
        else return __ldg(start + s);
    }
    // first attended token and attended length from the raw entries
    __device__ __forceinline__ int first_of(int st) const { return (kStart && st > 0) ? st : 0; }
    __device__ __forceinline__ int eff_of(int L, int st) const {
        const int Lc = clamp_len(L, cap);
        if constexpr (!kStart) {
            return Lc;
        } else {
            const int f = first_of(st);
            return f >= Lc ? 0 : Lc - f;
        }
    }
    __device__ __forceinline__ int first(int s) const { return first_of(raw_start(s)); }
    __device__ __forceinline__ int eff(int s) const { return eff_of(raw_len(s), raw_start(s)); }
};
template <int TT>
__device__ __forceinline__ int ntiles_of(int L) { return (L + TT - 1) / TT; }

// Entries [s0, s0 + E) of an int32 array (0 past n), all loads in flight together.
template <int E>
__device__ __forceinline__ void load_run(const int32_t* a, int s0, int n, int (&v)[E]) {
#pragma unroll
    for (int k = 0; k < E; ++k) v[k] = (s0 + k < n) ? __ldg(a + s0 + k) : 0;
}

// Sequences per lane in one round of the warp-wide length scans (256 per
// round).  A wider scan (32 per lane, 16-byte loads) was measured: its larger
// prologue made a cold-started tiny batch 8 us slower (instruction fetches)
// and it did not speed up a 2048-sequence batch.
constexpr int kScanPerLane = 8;

// Raw lengths (and starts) of the lane's sequences of the round at s0.
template <int E, class LN>
__device__ __forceinline__ void load_lens(const LN& ln, int s0, int (&v)[E], int (&st)[E]) {
    load_run<E>(ln.len, s0, ln.S, v);
    if constexpr (LN::kHasStart) {
        load_run<E>(ln.start, s0, ln.S, st);
    } else {
#pragma unroll
        for (int k = 0; k < E; ++k) st[k] = 0;
    }
}

// Warp-collective: total tiles W = units_per_seq * sum_s ceil(L_s / TT);
// *bad_len is set when some length is negative or overruns its table row.
template <int TT, int E = kScanPerLane, class LN>
__device__ inline int64_t total_tiles(const LN& ln, bool* bad_len = nullptr) {
    const int lane = threadIdx.x & 31;
    int64_t tot = 0;
    bool bad = false;
    for (int r0 = 0; r0 < ln.S; r0 += 32 * E) {
        const int s0 = r0 + lane * E;
        int v[E], st[E];
        load_lens<E>(ln, s0, v, st);
        int64_t part = 0;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            if (s0 + k < ln.S) {
                bad |= (v[k] < 0 || v[k] > ln.cap);
                part += ntiles_of<TT>(ln.eff_of(v[k], st[k]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(kFull, part, o);
        tot += part;
    }
    if (bad_len) *bad_len = __any_sync(kFull, bad);
    return tot * ln.units;
}

// Warp-collective: the total tiles W (as total_tiles) and the index of
// sequence s's first tile, in one pass over the lengths.
template <int TT, int E = kScanPerLane, class LN>
__device__ inline void seq_tile_base(const LN& ln, int s, int64_t* W, int64_t* base) {
    const int lane = threadIdx.x & 31;
    int64_t tot = 0, before = 0;
    for (int r0 = 0; r0 < ln.S; r0 += 32 * E) {
        const int s0 = r0 + lane * E;
        int v[E], st[E];
        load_lens<E>(ln, s0, v, st);
        int64_t part = 0, pb = 0;
#pragma unroll
        for (int k = 0; k < E; ++k) {
            const int64_t t = (s0 + k < ln.S) ? ntiles_of<TT>(ln.eff_of(v[k], st[k])) : 0;
            part += t;
            pb += s0 + k < s ? t : 0;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            part += __shfl_xor_sync(kFull, part, o);
            pb += __shfl_xor_sync(kFull, pb, o);
        }
        tot += part;
        before += pb;
    }
    *W = tot * ln.units;
    *base = before * ln.units;
}

struct SeqHit {
    int s;          // sequence holding tile P (num_seqs if none)
    int64_t base;   // index of its first tile
    int L;          // its raw seq_lens entry
    int st;         // its raw start entry (0 without starts)
};

// Warp-collective: the sequence whose tiles contain global tile P.
template <int TT, int E = kScanPerLane, class LN>
__device__ inline SeqHit find_seq(const LN& ln, int64_t P) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    for (int r0 = 0; r0 < ln.S; r0 += 32 * E) {
        const int s0 = r0 + lane * E;
        int v[E], st[E];
        load_lens<E>(ln, s0, v, st);
        int64_t part = 0;
#pragma unroll
        for (int k = 0; k < E; ++k)
            part += (s0 + k < ln.S) ? (int64_t)ntiles_of<TT>(ln.eff_of(v[k], st[k])) * ln.units : 0;
        int64_t incl = part;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += y;
        }
        const unsigned hit = __ballot_sync(kFull, base + incl > P);
        if (hit) {
            const int src = __ffs(hit) - 1;
            int found = 0, fl = 0, fst = 0;
            int64_t at = 0;
            if (lane == src) {
                int64_t acc = base + incl - part;
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const int64_t w = (s0 + k < ln.S) ? (int64_t)ntiles_of<TT>(ln.eff_of(v[k], st[k])) * ln.units : 0;
                    if (!found && acc + w > P) { found = s0 + k + 1; at = acc; fl = v[k]; fst = st[k]; }
                    acc += w;
                }
            }
            found = max(__shfl_sync(kFull, found, src) - 1, 0);
            at = __shfl_sync(kFull, at, src);
            fl = __shfl_sync(kFull, fl, src);
            fst = __shfl_sync(kFull, fst, src);
            return SeqHit{found, at, fl, fst};
        }
        base += __shfl_sync(kFull, incl, 31);
    }
    return SeqHit{ln.S, base, 0, 0};
}

// ----------------------------------------------------------------------------
// CTA-cooperative forms of the two scans: the CTA's threads share one pass
// over the lengths (kScanPerLane sequences per thread and round) instead of
// every warp walking all of them.  Every thread of the CTA must call them
// (they synchronise the CTA); blockDim.x is a multiple of 32, at most
// kScanThreads.
// ----------------------------------------------------------------------------
constexpr int kScanThreads = 256;
struct BlockScanSmem {
    int64_t ex[kScanThreads];        // per-thread exclusive tile prefix of a round
    int64_t wsum[kScanThreads / 32]; // per-warp sums
};

// Exclusive prefix of v over the CTA's threads in thread order; *total is
// the CTA's sum.  The caller synchronises before the next call.
__device__ __forceinline__ int64_t block_excl_sum(int64_t v, BlockScanSmem& sm, int64_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) sm.wsum[warp] = incl;
    __syncthreads();
    int64_t before = 0, tot = 0;
    for (int w = 0; w < nw; ++w) {
        const int64_t x = sm.wsum[w];
        before += (w < warp) ? x : 0;
        tot += x;
    }
    *total = tot;
    return before + incl - v;
}

// CTA-collective total_tiles.
template <int TT, class LN>
__device__ inline int64_t block_total_tiles(const LN& ln, BlockScanSmem& sm, bool* bad_len = nullptr) {
    constexpr int E = kScanPerLane;
    int64_t part = 0;
    bool bad = false;
    for (int r0 = 0; r0 < ln.S; r0 += blockDim.x * E) {
        const int s0 = r0 + threadIdx.x * E;
        int v[E], st[E];
        load_lens<E>(ln, s0, v, st);
#pragma unroll
        for (int k = 0; k < E; ++k) {
            if (s0 + k < ln.S) {
                bad |= (v[k] < 0 || v[k] > ln.cap);
                part += ntiles_of<TT>(ln.eff_of(v[k], st[k]));
            }
        }
    }
    int64_t tot;
    block_excl_sum(part, sm, &tot);
    const int any_bad = __syncthreads_or(bad);  // also: every thread has read the warp sums
    if (bad_len) *bad_len = any_bad != 0;
    return tot * ln.units;
}

// CTA-collective find_seq: each warp passes its own tile P and gets the
// sequence whose tiles contain it (s = num_seqs when P is past the last).
template <int TT, class LN>
__device__ inline SeqHit block_find_seq(const LN& ln, int64_t P, BlockScanSmem& sm) {
    constexpr int E = kScanPerLane;
    static_assert(E <= 32, "one sequence per lane in the final step");
    const int lane = threadIdx.x & 31;
    SeqHit hit{ln.S, 0, 0, 0};
    bool found = false;
    int64_t base = 0;
    for (int r0 = 0; r0 < ln.S; r0 += blockDim.x * E) {
        const int s0 = r0 + threadIdx.x * E;
        int v[E], st[E];
        load_lens<E>(ln, s0, v, st);
        int64_t cnt = 0;
#pragma unroll
        for (int k = 0; k < E; ++k)
            cnt += (s0 + k < ln.S) ? (int64_t)ntiles_of<TT>(ln.eff_of(v[k], st[k])) * ln.units : 0;
        int64_t tot;
        sm.ex[threadIdx.x] = base + block_excl_sum(cnt, sm, &tot);
        __syncthreads();
        if (!found && P < base + tot) {  // warp-uniform
            // the last thread t with ex[t] <= P holds tile P (ex does not decrease)
            int t = 0;
            for (int c0 = 0; c0 < (int)blockDim.x; c0 += 32) {
                const unsigned le = __ballot_sync(kFull, sm.ex[c0 + lane] <= P);
                if (le) t = c0 + 31 - __clz(le);
                if (le != kFull) break;
            }
            // thread t's sequences, one per lane
            const int s = r0 + t * E + lane;
            const bool in = lane < E && s < ln.S;
            const int L = in ? ln.raw_len(s) : 0;
            const int sst = in ? ln.raw_start(s) : 0;
            const int64_t w = in ? (int64_t)ntiles_of<TT>(ln.eff_of(L, sst)) * ln.units : 0;
            int64_t incl = w;
#pragma unroll
            for (int o = 1; o < E; o <<= 1) {
                const int64_t y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            const int64_t at = sm.ex[t] + incl - w;
            const unsigned h = __ballot_sync(kFull, in && at + w > P);
            const int src = __ffs(h) - 1;  // h != 0: thread t's sequences hold P
            hit = SeqHit{__shfl_sync(kFull, s, src), __shfl_sync(kFull, at, src), __shfl_sync(kFull, L, src),
                         __shfl_sync(kFull, sst, src)};
            found = true;
        }
        base += tot;
        __syncthreads();  // ex and the warp sums are rewritten by the next round
    }
    if (!found) hit.base = base;
    return hit;
}

// First attended token of the walk's current sequence: a field only when
// ranges may start past token 0.
template <bool kStart> struct WalkStart { int st; int nst; };
template <> struct WalkStart<false> { static constexpr int st = 0; };

// Walk over a worker's tiles (TT tokens each) in order: (sequence, unit j, tile i).
// The raw entries of the next sequence are loaded when the walk enters a
// sequence, so moving on does not wait for a load.
template <int TT, bool kStart = false>
struct Walk : WalkStart<kStart> {
    int s, L, nt, j, i, seg_i0, ord;  // L: attended length
    int nl;                           // raw seq_lens entry of sequence s + 1 (prefetched)
    int64_t T, te;
    bool done;

    __device__ void prefetch_next(const Lens<kStart>& ln) {
        const bool in = s + 1 < ln.S;
        nl = in ? ln.raw_len(s + 1) : 0;
        if constexpr (kStart) this->nst = in ? ln.raw_start(s + 1) : 0;
    }
    __device__ void init(const Lens<kStart>& ln, int64_t tb, int64_t te_) {
        init(ln, tb, te_, tb < te_ ? find_seq<TT>(ln, tb) : SeqHit{ln.S, 0, 0, 0});
    }
    // h: the sequence holding tile tb (find_seq or block_find_seq)
    __device__ void init(const Lens<kStart>& ln, int64_t tb, int64_t te_, const SeqHit& h) {
        te = te_;
        T = tb;
        done = tb >= te_;
        ord = 0;
        s = 0; L = 0; nt = 1; j = 0; i = 0; seg_i0 = 0; nl = 0;
        if constexpr (kStart) { this->st = 0; this->nst = 0; }
        if (done) return;
        s = h.s;
        L = ln.eff_of(h.L, h.st);
        if constexpr (kStart) this->st = ln.first_of(h.st);
        nt = ntiles_of<TT>(L);
        j = (int)((tb - h.base) / nt);
        i = (int)((tb - h.base) % nt);
        seg_i0 = i;
        prefetch_next(ln);
    }
    __device__ bool first() const { return i == seg_i0; }
    __device__ bool last() const { return i == nt - 1 || T == te - 1; }
    __device__ void advance(const Lens<kStart>& ln) {
        if (done) return;
        if (++T >= te) { done = true; return; }
        if (++i == nt) {
            i = 0;
            seg_i0 = 0;
            ++ord;
            if (++j == ln.units) {
                j = 0;
                do {  // a later non-empty sequence exists because T < te <= W
                    ++s;
                    if (s < ln.S) {
                        int nst = 0;
                        if constexpr (kStart) nst = this->nst;
                        L = ln.eff_of(nl, nst);
                        if constexpr (kStart) this->st = ln.first_of(nst);
                        prefetch_next(ln);
                    } else {
                        L = TT;
                        if constexpr (kStart) this->st = 0;
                    }
                    nt = ntiles_of<TT>(L);
                } while (nt == 0);
            }
        }
    }
};

// ----------------------------------------------------------------------------
// Per-variant traits.
// ----------------------------------------------------------------------------
enum class Path { kMma16, kFp8, kF32 };

// kQH_: q heads one q slot holds (>= the unit's heads, min(g, 8)); a slot per
// ring stage, since the issue walk may be up to kStages-1 units ahead.
template <typename KvT, typename QT, int D_, Path P_, int kWarps_, int kStages_, int kTT_ = kTileTokens,
          int kQH_ = kHeadsPerUnit>
struct Cfg {
    using kv_t = KvT;
    using q_t = QT;
    static constexpr Path kPath = P_;
    static constexpr int D = D_;
    static constexpr int kWarps = kWarps_;
    static constexpr int kStages = kStages_;
    static constexpr int kTT = kTT_;                    // tokens per tile
    static constexpr int kSubBytes = kTT * 128;         // one 128-byte-wide column of a tile
    static constexpr int kKvBytes = (int)sizeof(KvT);
    static constexpr int kQBytes = (int)sizeof(QT);
    static constexpr int kRowBytes = D * kKvBytes;
    static constexpr int kNSub = kRowBytes / 128;       // 128-byte columns per row
    static constexpr int kTensorTile = kNSub * kSubBytes;
    static constexpr int kStageBytes = 2 * kTensorTile; // K tile + V tile
    static constexpr int kQH = kQH_;
    static constexpr int kQSlot = kQH * D * kQBytes;
    static constexpr int kWarpBytes = kStages * (kStageBytes + kQSlot);
    static constexpr int kSmemBytes = kWarps * kWarpBytes + 1024;  // + alignment slack
    static constexpr int kChunksPerRow = kRowBytes / 16;
    static constexpr int kRowsPerInst = 32 / kChunksPerRow;         // rows one warp-wide cp.async covers
    static_assert(16 % kRowsPerInst == 0, "a cp.async row group never straddles a 16-token block");
    static_assert(kTT == 16 || (kTT == 32 && P_ != Path::kF32), "tile sizes");
    static_assert(kRowBytes % 128 == 0, "rows must be whole 128-byte columns");
    // the swizzle only needs each tile and q slot on a 128-byte boundary
    static_assert(kStageBytes % 128 == 0 && kQSlot % 128 == 0, "128-byte stage alignment");
    static_assert(kQH >= 1 && kQH <= kHeadsPerUnit, "q slot heads");
    static_assert(kWarps <= kMaxWarpsPerCta, "workspace sizing");
};

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Zero rows [valid, TT) of a V tile (NSUB columns of TT x 128 B).  Used on a
// sequence's last tile (FP8 decode tiles, the cascade prefix pass) so the
// unused slots (never written, any bits) cannot reach the tensor-core P.V
// product; 16-bit decode tiles zero-fill those rows as they load them.
template <int kNSub, int TT>
__device__ __forceinline__ void zero_tail_rows(uint8_t* tile, int valid, int lane) {
    constexpr int kSubBytes = TT * 128;
    const int rows = TT - valid;
    const int per_sub = rows * 8;  // 16-byte chunks
    for (int idx = lane; idx < kNSub * per_sub; idx += 32) {
        const int sub = idx / per_sub, rem = idx % per_sub;
        const int row = valid + rem / 8, ch = rem % 8;
        *reinterpret_cast<uint4*>(tile + sub * kSubBytes + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
}

// Swizzled byte offset of 16-byte chunk `c` (of the whole row) of token row t
// in a tile: column c/8, line t, chunk (c%8) XOR (t%8) -- conflict-free for
// the ldmatrix / 16-byte shared loads below and for the cp.async writes.
template <int TT = kTileTokens>
__device__ __forceinline__ uint32_t sw_off(int t, int c) {
    return (uint32_t)((c >> 3) * (TT * 128) + t * 128 + ((((c & 7) ^ t) & 7) << 4));
}

// Output / workspace sink of one unit segment.
struct Sink {
    bool split;
    bool part;     // whole unit, result to part_o / part_ml (read only when kPart)
    int64_t seg;   // workspace segment (split only)
    int64_t row0;  // output row (s * Hq + first head of the chunk)
    int nh;
};

// kPart: the cascade suffix pass, whose whole units may be partials.
template <typename QT, bool kPart>
__device__ __forceinline__ void sink_write(const DecodeParams& p, const SuffixArg<kPart>& sx, const Sink& k,
                                           int D, int h, int d, float o, float l, float vscale) {
    if (h >= k.nh) return;
    if constexpr (kPart) {
        if (k.part) {
            sx.part_o[(k.row0 + h) * D + d] = o * vscale;
            return;
        }
    }
    if (!k.split) {
        QT* out = reinterpret_cast<QT*>(p.out) + (k.row0 + h) * D + d;
        *out = from_f32<QT>(l > 0.f ? o * vscale / l : 0.f);
    } else {
        p.ws_o[(k.seg * p.hpu + h) * D + d] = o * vscale;
    }
}

// ---- 16-bit caches (f16 / bf16) and FP8 caches: tensor-core tile math --------
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
    // This lane's swizzled byte offsets inside a tile, fixed for the kernel:
    // 16-bit path: ldmatrix row addresses of k-step / head_dim tile k4 (mod 4)
    // of the first 16 tokens (later k-steps add a 128-byte column block,
    // later 16-token m-tiles add 2 KB); FP8 path: the 16-byte K and V chunks
    // the lane reads for its first rows.
    uint32_t ko[4], vo[4];

    __device__ void init_lane() {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        if constexpr (!kFp8) {
            const int r = lane & 7, mtx = lane >> 3;
            const int tk = r + ((mtx & 1) << 3), tv = r + ((mtx >> 1) << 3);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                ko[k4] = sw_off<C::kTT>(tk, 2 * k4 + (mtx >> 1));
                vo[k4] = sw_off<C::kTT>(tv, 2 * k4 + (mtx & 1));
            }
        } else {
            ko[0] = sw_off<C::kTT>(gid, 2 * tig);
            ko[1] = sw_off<C::kTT>(gid, 2 * tig + 1);
            vo[0] = sw_off<C::kTT>(2 * tig, gid);
            vo[1] = sw_off<C::kTT>(2 * tig + 1, gid);
            ko[2] = ko[3] = vo[2] = vo[3] = 0;
        }
    }

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

    // One tile of TT = 16 * NM tokens: S^T per 16-token m-tile, one online
    // softmax step over the whole tile, then P.V with one k-step per m-tile.
    __device__ void tile(uint8_t* kt, uint8_t* vt, int valid) {
        constexpr int TT = C::kTT, NM = TT / 16;
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        // rows >= valid: zero-filled by issue_tile for 16-bit caches; FP8
        // codes are loaded as stored and zeroed here, so that unused slots
        // (never written, any bits) cannot reach the P.V product
        if constexpr (C::kPath == Path::kFp8)
            if (valid < TT) zero_tail_rows<C::kNSub, TT>(vt, valid, lane);
        const uint32_t kb = smem_u32(kt), vb = smem_u32(vt);
        float x[NM][4];
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (!kFp8) {
                // row t = 16m + (lane's row): the XOR part of the swizzle only
                // sees t mod 8, so m and the column block are plain offsets
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    uint32_t a[4];
                    ldsm_x4(a, kb + ko[kk & 3] + (kk >> 2) * (TT * 128) + m * 2048);
                    if (kk & 1) mma16816<kOpBf16>(sb, a, qf[kk][0], qf[kk][1]);
                    else        mma16816<kOpBf16>(sa, a, qf[kk][0], qf[kk][1]);
                }
            } else {
                // K rows gid and gid+8 of the m-tile, bytes [32*tig, 32*tig+32).
                const uint4 r0a = *reinterpret_cast<const uint4*>(kt + ko[0] + m * 2048);
                const uint4 r0b = *reinterpret_cast<const uint4*>(kt + ko[1] + m * 2048);
                const uint4 r1a = *reinterpret_cast<const uint4*>(kt + ko[0] + m * 2048 + 1024);
                const uint4 r1b = *reinterpret_cast<const uint4*>(kt + ko[1] + m * 2048 + 1024);
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
            x[m][0] = (sa[0] + sb[0]) * sl0; x[m][1] = (sa[1] + sb[1]) * sl1;
            x[m][2] = (sa[2] + sb[2]) * sl0; x[m][3] = (sa[3] + sb[3]) * sl1;
            if (16 * m + gid >= valid) x[m][0] = x[m][1] = -INFINITY;
            if (16 * m + gid + 8 >= valid) x[m][2] = x[m][3] = -INFINITY;
        }
        float mx0 = fmaxf(x[0][0], x[0][2]), mx1 = fmaxf(x[0][1], x[0][3]);
#pragma unroll
        for (int m = 1; m < NM; ++m) {
            mx0 = fmaxf(mx0, fmaxf(x[m][0], x[m][2]));
            mx1 = fmaxf(mx1, fmaxf(x[m][1], x[m][3]));
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
        }
        // Lazy rescale: a head's reference maximum moves only when the tile's
        // maximum passes it by more than 2^kLazyLog2 (then the whole warp
        // rescales o and l at once); otherwise P = 2^(x - m) <= 2^kLazyLog2,
        // still exact in its 16-bit parts, and o, l stay relative to the same
        // m (the sinks and the (m, l) merge accept any reference).
        constexpr float kLazyLog2 = 8.f;
        if (__any_sync(kFull, mx0 > m0 + kLazyLog2 || mx1 > m1 + kLazyLog2)) {
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            l0 *= al0;
            l1 *= al1;
#pragma unroll
            for (int mi = 0; mi < MT; ++mi) {
                acc[mi][0] *= al0; acc[mi][1] *= al1; acc[mi][2] *= al0; acc[mi][3] *= al1;
            }
        }
        // P goes to the tensor core in the V operand's 16-bit type.  bf16 keeps
        // only 8 significant bits, so for bf16 caches P is carried as
        // hi + lo bf16 parts (two products, ~16 significant bits): the P.V sum
        // then matches fp32 P to well inside the tolerance.  f16 (11 bits) and
        // the FP8 path (f16) use one part.
        uint32_t b0[NM], b1[NM], c0[NM], c1[NM];
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            const float e0 = ex2(x[m][0] - m0), e1 = ex2(x[m][1] - m1);
            const float e2 = ex2(x[m][2] - m0), e3 = ex2(x[m][3] - m1);
            const uint32_t X0 = pack2<kOpBf16>(e0, e1);
            const uint32_t X1 = pack2<kOpBf16>(e2, e3);
            if constexpr (kOpBf16) {
                const float2 h0 = unpack2<true>(X0), h1 = unpack2<true>(X1);
                c0[m] = movm_trans(pack2<true>(e0 - h0.x, e1 - h0.y));
                c1[m] = movm_trans(pack2<true>(e2 - h1.x, e3 - h1.y));
                ls0 += e0 + e2;
                ls1 += e1 + e3;
            } else {
                const float2 p0 = unpack2<false>(X0), p1 = unpack2<false>(X1);
                ls0 += p0.x + p1.x;  // normaliser from the rounded P actually used
                ls1 += p0.y + p1.y;
                c0[m] = c1[m] = 0u;
            }
            b0[m] = movm_trans(X0);  // P^T as mma B
            b1[m] = movm_trans(X1);
        }
        l0 += ls0;
        l1 += ls1;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            if constexpr (!kFp8) {
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    uint32_t a[4];
                    ldsm_x4_trans(a, vb + vo[mi & 3] + (mi >> 2) * (TT * 128) + m * 2048);
                    mma16816<kOpBf16>(acc[mi], a, b0[m], b1[m]);
                    if constexpr (kOpBf16) mma16816<true>(acc[mi], a, c0[m], c1[m]);
                }
            } else {
                // V^T fragments: thread gid owns d in [16*gid, 16*gid+16) (one chunk),
                // rows 2tig, 2tig+1, 2tig+8, 2tig+9 of the m-tile; m-tile mi covers
                // d = 16*gid + 2*mi (row gid) and 16*gid + 2*mi + 1 (row gid+8).
                const uint4 R0 = *reinterpret_cast<const uint4*>(vt + vo[0] + m * 2048);
                const uint4 R1 = *reinterpret_cast<const uint4*>(vt + vo[1] + m * 2048);
                const uint4 R8 = *reinterpret_cast<const uint4*>(vt + vo[0] + m * 2048 + 1024);
                const uint4 R9 = *reinterpret_cast<const uint4*>(vt + vo[1] + m * 2048 + 1024);
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
                    mma16816<false>(acc[2 * w], a, b0[m], b1[m]);
                    a[0] = e4m3x2_to_f16x2((uint16_t)(Y & 0xffffu));
                    a[1] = e4m3x2_to_f16x2((uint16_t)(Y >> 16));
                    a[2] = e4m3x2_to_f16x2((uint16_t)(Y8 & 0xffffu));
                    a[3] = e4m3x2_to_f16x2((uint16_t)(Y8 >> 16));
                    mma16816<false>(acc[2 * w + 1], a, b0[m], b1[m]);
                }
            }
        }
    }

    // End of a unit segment: the output (whole unit) or a partial (split).
    template <bool kPart>
    __device__ void finish(const DecodeParams& p, const SuffixArg<kPart>& sx, const Sink& k, float vscale) {
        using QT = typename C::q_t;
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
        float a0 = l0, a1 = l1;
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            a0 += __shfl_xor_sync(kFull, a0, o);
            a1 += __shfl_xor_sync(kFull, a1, o);
        }
        const int h0 = 2 * tig, h1 = 2 * tig + 1;
        bool to_out = !k.split;
        if constexpr (kPart) to_out = to_out && !k.part;
        if (to_out) {
            // the output rows, normalised and rounded RNE to the q dtype, two
            // adjacent head_dim elements per 32-bit store
            constexpr bool kQb = std::is_same<QT, __nv_bfloat16>::value;
            const float s0 = a0 > 0.f ? vscale / a0 : 0.f, s1 = a1 > 0.f ? vscale / a1 : 0.f;
            QT* out = reinterpret_cast<QT*>(p.out) + k.row0 * D;
            if constexpr (!kFp8) {
                // O^T fragments hold (d = 16 mi + gid (+8), heads 2 tig, 2 tig + 1):
                // transposed, lane (gid, tig) holds head gid at d = 2 tig, 2 tig + 1
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    const uint32_t lo = movm_trans(pack2<kQb>(acc[mi][0] * s0, acc[mi][1] * s1));
                    const uint32_t hi = movm_trans(pack2<kQb>(acc[mi][2] * s0, acc[mi][3] * s1));
                    if (gid < k.nh) {
                        *reinterpret_cast<uint32_t*>(out + gid * D + 16 * mi + 2 * tig) = lo;
                        *reinterpret_cast<uint32_t*>(out + gid * D + 16 * mi + 8 + 2 * tig) = hi;
                    }
                }
            } else {
                // FP8 path: lane holds d = 16 gid + 2 mi and the next one of heads h0, h1
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    if (h0 < k.nh)
                        *reinterpret_cast<uint32_t*>(out + h0 * D + 16 * gid + 2 * mi) =
                            pack2<kQb>(acc[mi][0] * s0, acc[mi][2] * s0);
                    if (h1 < k.nh)
                        *reinterpret_cast<uint32_t*>(out + h1 * D + 16 * gid + 2 * mi) =
                            pack2<kQb>(acc[mi][1] * s1, acc[mi][3] * s1);
                }
            }
            return;
        }
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
            int d0, d1;
            if constexpr (!kFp8) { d0 = 16 * mi + gid; d1 = d0 + 8; }
            else { d0 = 16 * gid + 2 * mi; d1 = d0 + 1; }
            sink_write<QT, kPart>(p, sx, k, D, h0, d0, acc[mi][0], a0, vscale);
            sink_write<QT, kPart>(p, sx, k, D, h1, d0, acc[mi][1], a1, vscale);
            sink_write<QT, kPart>(p, sx, k, D, h0, d1, acc[mi][2], a0, vscale);
            sink_write<QT, kPart>(p, sx, k, D, h1, d1, acc[mi][3], a1, vscale);
        }
        if constexpr (kPart) {
            if (gid == 0 && (k.split || k.part)) {
                float2* ml = k.part ? sx.part_ml + k.row0 : p.ws_ml + k.seg * p.hpu;
                if (h0 < k.nh) ml[h0] = make_float2(m0, a0);
                if (h1 < k.nh) ml[h1] = make_float2(m1, a1);
            }
        } else if (k.split && gid == 0) {
            if (h0 < k.nh) p.ws_ml[k.seg * p.hpu + h0] = make_float2(m0, a0);
            if (h1 < k.nh) p.ws_ml[k.seg * p.hpu + h1] = make_float2(m1, a1);
        }
    }
};

// ---- fp32 caches: CUDA-core tile math ---------------------------------------
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
    __device__ void init_lane() {}
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
    template <bool kPart>
    __device__ void finish(const DecodeParams& p, const SuffixArg<kPart>& sx, const Sink& k, float vscale) {
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
            if (rh == 0) {
                sink_write<float, kPart>(p, sx, k, D, h, 4 * c + 0, a.x, ls, vscale);
                sink_write<float, kPart>(p, sx, k, D, h, 4 * c + 1, a.y, ls, vscale);
                sink_write<float, kPart>(p, sx, k, D, h, 4 * c + 2, a.z, ls, vscale);
                sink_write<float, kPart>(p, sx, k, D, h, 4 * c + 3, a.w, ls, vscale);
            }
            if constexpr (kPart) {
                if (lane == 0 && h < k.nh) {
                    if (k.part) sx.part_ml[k.row0 + h] = make_float2(m[h], ls);
                    else if (k.split) p.ws_ml[k.seg * p.hpu + h] = make_float2(m[h], ls);
                }
            } else if (k.split && lane == 0 && h < k.nh) {
                p.ws_ml[k.seg * p.hpu + h] = make_float2(m[h], ls);
            }
        }
    }
};

template <class C>
using ConsumerOf = typename std::conditional<C::kPath == Path::kF32, F32Consumer<C>, MmaConsumer<C>>::type;

// ----------------------------------------------------------------------------
// Block-table prefetcher of one warp: entries [base, base+64) of the current
// sequence's row in two registers per lane, the second batch fetched while
// the first is in use.
// ----------------------------------------------------------------------------
struct TablePrefetch {
    int s = -1, base = 0, cur = 0, nxt = 0;

    __device__ int get(const DecodeParams& p, int seq, int b, int nblk, int lane) {
        const int32_t* row = p.block_tables + (int64_t)seq * p.max_blocks_per_seq;
        if (seq != s || b < base || b >= base + 64) {
            s = seq;
            base = b;
            cur = (b + lane < nblk) ? __ldg(row + b + lane) : 0;
            nxt = (b + 32 + lane < nblk) ? __ldg(row + b + 32 + lane) : 0;
        } else if (b >= base + 32) {
            base += 32;
            cur = nxt;
            nxt = (base + 32 + lane < nblk) ? __ldg(row + base + 32 + lane) : 0;
        }
        return __shfl_sync(kFull, cur, b - base);
    }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// n = 16 copies the chunk, n = 0 writes 16 zero bytes and reads nothing
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// kv head and head chunk of unit j (no division in the common nch == 1 case)
__device__ __forceinline__ int2 unit_head(int j, int nch) {
    if (nch == 1) return make_int2(j, 0);
    const int kh = j / nch;
    return make_int2(kh, j - kh * nch);
}

// This lane's part of a tile's cp.async loads, fixed for the kernel: the
// swizzled shared-memory offsets of its rows (the swizzle repeats every 8
// rows, so kP offsets cover a tile; later row groups add 1 KB each) and its
// byte offset inside a row group of the cache.
template <class C>
struct IssueLane {
    static constexpr int kR = C::kRowsPerInst;
    static constexpr int kP = 8 / kR;      // distinct swizzle patterns
    uint32_t so[kP];
    int64_t goff;                          // r0 * row_stride + 16 * cr
    int64_t gstep;                         // kR * row_stride
    int r0;                                // the lane's row within each instruction's kR rows
    __device__ void init(const DecodeParams& p) {
        const int lane = threadIdx.x & 31;
        const int cr = lane % C::kChunksPerRow;
        r0 = lane / C::kChunksPerRow;
#pragma unroll
        for (int k = 0; k < kP; ++k) so[k] = sw_off<C::kTT>(k * kR + r0, cr);
        const int64_t row_stride = (int64_t)p.num_kv_heads * C::kRowBytes;  // bytes between tokens
        goff = r0 * row_stride + 16 * cr;
        gstep = kR * row_stride;
    }
};

// Issue the async loads of the walk's current tile (and, on a unit's first
// tile, of its q rows) into stage `stg` / q slot `qslot`.  lg_bs: log2 of
// the block size (16 or 32 tokens).
template <class C, bool kStart>
__device__ __forceinline__ void issue_tile(const DecodeParams& p, const Walk<C::kTT, kStart>& w, TablePrefetch& tp,
                                           const IssueLane<C>& il, int lg_bs, uint8_t* stg, uint8_t* qslot) {
    const int lane = threadIdx.x & 31;
    const int2 hc = unit_head(w.j, p.nch);
    const int kh = hc.x, c = hc.y;
    const int tok = w.st + w.i * C::kTT;  // absolute token of the tile's first row (a multiple of 16)
    const int bmask = (1 << lg_bs) - 1;
    const int nblk = (w.st + w.L + bmask) >> lg_bs;
    const int b0 = tok >> lg_bs;
    auto checked = [&](int ph) {
        if (ph < 0 || ph >= p.num_blocks) {
            if (lane == 0) raise_error(p.err, PKV_DEVERR_BLOCK_ID);
            ph = 0;
        }
        return ph;
    };
    const int phys0 = checked(tp.get(p, w.s, b0, nblk, lane));
    const int64_t kv_row = (int64_t)p.num_kv_heads * C::kRowBytes;  // bytes between tokens
    const int64_t base0 = ((((int64_t)phys0 << lg_bs) + (tok & bmask)) * p.num_kv_heads + kh) * C::kRowBytes;
    // A 32-token tile over 16-token blocks covers two blocks: rows 16.. come
    // from the next one (or, past the sequence's last block, again from the
    // first: those rows are masked).  base1 is offset so that row t reads
    // base1 + t * row_stride.
    int64_t base1 = base0;
    if constexpr (C::kTT > 16) {
        if (lg_bs == 4) {
            const int phys1 = b0 + 1 < nblk ? checked(tp.get(p, w.s, b0 + 1, nblk, lane)) : phys0;
            base1 = (((int64_t)phys1 << lg_bs) * p.num_kv_heads + kh) * C::kRowBytes - 16 * kv_row;
        }
    }
    const uint32_t kdst = smem_u32(stg), vdst = smem_u32(stg + C::kTensorTile);
    const uint8_t* kl = p.key_cache + il.goff;
    const uint8_t* vl = p.value_cache + il.goff;
    // rows of the tile inside the sequence (16-bit caches zero-fill the rest:
    // measured faster there; the FP8 and fp32 tiles mask or zero them after
    // the load, which keeps their kernels' code and registers smaller)
    const int nvalid = C::kPath == Path::kMma16 ? w.L - w.i * C::kTT : C::kTT;
    if (nvalid >= C::kTT) {
#pragma unroll
        for (int it = 0; it < C::kTT / C::kRowsPerInst; ++it) {
            // rows >= 16 exactly when it * kRowsPerInst >= 16
            const int64_t off = (it * C::kRowsPerInst >= 16 ? base1 : base0) + it * il.gstep;
            const uint32_t so = il.so[it % IssueLane<C>::kP] + (it / IssueLane<C>::kP) * 1024;
            cp_async16(kdst + so, kl + off);
            cp_async16(vdst + so, vl + off);
        }
    } else {
        // the sequence's last, partly filled tile: rows past its end are
        // zero-filled in shared memory and not read (their addresses stay
        // inside the block, or the first block of the tile)
#pragma unroll
        for (int it = 0; it < C::kTT / C::kRowsPerInst; ++it) {
            const int64_t off = (it * C::kRowsPerInst >= 16 ? base1 : base0) + it * il.gstep;
            const uint32_t so = il.so[it % IssueLane<C>::kP] + (it / IssueLane<C>::kP) * 1024;
            const uint32_t n = it * C::kRowsPerInst + il.r0 < nvalid ? 16u : 0u;
            cp_async16_zfill(kdst + so, kl + off, n);
            cp_async16_zfill(vdst + so, vl + off, n);
        }
    }
    if (w.first()) {
        const int nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
        const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(p.q) +
            ((int64_t)w.s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c) * C::D * C::kQBytes;
        const int chunks = nh * C::D * C::kQBytes / 16;
        for (int ch = lane; ch < chunks; ch += 32) cp_async16(smem_u32(qslot + ch * 16), qsrc + ch * 16);
    }
}

// ----------------------------------------------------------------------------
// The kernel: every warp is an independent worker.
// ----------------------------------------------------------------------------
// kSuffix: the cascade suffix pass (per-sequence start tokens, partial
// output); false compiles the plain decode path without either.
// The cascade suffix pass is a programmatic dependent of the prefix pass,
// whose results it does not read: it may run beside the prefix pass's last
// CTAs, but it completes only after that grid, so that the passes after it
// see every prefix partial.  Every exit of a suffix CTA waits.
template <bool kSuffix>
struct WaitPrimaryAtExit {
    __device__ ~WaitPrimaryAtExit() {
        if constexpr (kSuffix) asm volatile("griddepcontrol.wait;" ::: "memory");
    }
};

// kWideScan: the CTA-wide length scans (batches that one round of a warp's
// scan does not cover); false: each warp scans alone, with no CTA barrier.
// Two instantiations rather than a branch: with the CTA-wide form compiled
// in, a cold-started tiny batch measured 4 us slower.
template <class C, bool kSuffix, bool kWideScan>
__global__ void __launch_bounds__(C::kWarps * 32, 1)
pkv_decode_kernel(const DecodeParams p, const SuffixArg<kSuffix> sx) {
    const WaitPrimaryAtExit<kSuffix> wait_at_exit;
    // let the merge grid (a programmatic dependent launch) be scheduled now:
    // its CTAs locate their units while this grid runs and wait for its
    // completion before reading any partial result
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t* stages = smem + warp * C::kWarpBytes;
    uint8_t* qslots = stages + C::kStages * C::kStageBytes;

    const Lens<kSuffix> ln{p.seq_lens, sx.seq_start, p.num_seqs, p.num_kv_heads * p.nch,
                           p.max_blocks_per_seq * p.block_size};
    int64_t workers = (int64_t)gridDim.x * C::kWarps;
    int64_t cta = blockIdx.x;
    if constexpr (kSuffix) {
        if (sx.prefix_tile > 0) {
            // beside the prefix pass the CTAs do not start in index order
            // (some wait for a prefix CTA's SM): the first to arrive take the
            // worker slots, so the pass's share runs on the SMs free first
            __shared__ int slot;
            if (threadIdx.x == 0) slot = atomicAdd(sx.cta_ticket, 1);
            __syncthreads();
            cta = slot;
        }
    }
    const int64_t wid = cta * C::kWarps + warp;
    // the cascade suffix pass beside the prefix pass: this pass's share of
    // the grid (the warps past it find no tiles and leave)
    auto side_by_side = [&](int64_t Wsuf) {
        if constexpr (kSuffix) {
            if (sx.prefix_tile > 0) {
                const int64_t Wp = cascade_prefix_tiles(sx.prefix_eff, sx.num_groups, sx.prefix_units, sx.prefix_tile);
                workers = (int64_t)(gridDim.x - cascade_prefix_ctas(Wp, sx.prefix_tile, Wsuf, C::kTT, gridDim.x)) *
                          C::kWarps;
            }
        }
    };
    // the total and every warp's first tile
    bool bad_len = false;
    int64_t W, tb, te;
    Walk<C::kTT, kSuffix> iw, cw;  // issue walk (runs kStages-1 tiles ahead) and compute walk
    if constexpr (!kWideScan) {
        W = total_tiles<C::kTT>(ln, &bad_len);
        side_by_side(W);
        const int64_t chunk = (W + workers - 1) / workers;
        tb = min(W, wid * chunk);
        te = min(W, tb + chunk);
        if (tb < te) iw.init(ln, tb, te);
    } else {
        __shared__ BlockScanSmem scan_sm;  // one pass over the lengths per CTA
        W = block_total_tiles<C::kTT>(ln, scan_sm, &bad_len);
        side_by_side(W);
        const int64_t chunk = (W + workers - 1) / workers;
        tb = min(W, wid * chunk);
        te = min(W, tb + chunk);
        const SeqHit hit = block_find_seq<C::kTT>(ln, tb, scan_sm);  // every warp takes part
        if (tb < te) iw.init(ln, tb, te, hit);
    }
    if (bad_len && wid == 0 && lane == 0) raise_error(p.err, PKV_DEVERR_SEQ_LEN);
    if (tb >= te) return;

    cw = iw;
    TablePrefetch tp;
    IssueLane<C> il;
    il.init(p);
    const int lg_bs = 31 - __clz(p.block_size);
#pragma unroll 1
    for (int k = 0; k < C::kStages - 1; ++k) {
        if (!iw.done)
            issue_tile<C>(p, iw, tp, il, lg_bs, stages + k * C::kStageBytes, qslots + (iw.ord % C::kStages) * C::kQSlot);
        cp_async_commit();
        iw.advance(ln);
    }
    const float kscale = (C::kPath == Path::kFp8 && p.k_scale) ? __ldg(p.k_scale) : 1.f;
    const float vscale = (C::kPath == Path::kFp8 && p.v_scale) ? __ldg(p.v_scale) : 1.f;
    ConsumerOf<C> cs;
    cs.init_lane();
#pragma unroll 1
    for (int n = 0; !cw.done; ++n) {
        if (!iw.done)
            issue_tile<C>(p, iw, tp, il, lg_bs, stages + ((n + C::kStages - 1) % C::kStages) * C::kStageBytes,
                          qslots + (iw.ord % C::kStages) * C::kQSlot);
        cp_async_commit();
        iw.advance(ln);
        cp_async_wait<C::kStages - 1>();
        __syncwarp();
        const int2 hc = unit_head(cw.j, p.nch);
        const int kh = hc.x, c = hc.y;
        const int nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
        if (cw.first()) {
            cs.load_q(qslots + (cw.ord % C::kStages) * C::kQSlot, nh, p.scale_log2, kscale);
            cs.reset();
        }
        uint8_t* kt = stages + (n % C::kStages) * C::kStageBytes;
        cs.tile(kt, kt + C::kTensorTile, min(C::kTT, cw.L - cw.i * C::kTT));
        if (cw.last()) {
            Sink k;
            k.split = (cw.seg_i0 != 0) || (cw.i != cw.nt - 1);
            k.part = kSuffix && !k.split && cw.st > 0;
            k.seg = wid + ((int64_t)cw.s * p.num_kv_heads + kh) * p.nch + c;
            k.row0 = (int64_t)cw.s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c;
            k.nh = nh;
            cs.template finish<kSuffix>(p, sx, k, vscale);
        }
        __syncwarp();  // every lane is done with this stage before it is refilled
        cw.advance(ln);
    }
    cp_async_wait<0>();
}

// ----------------------------------------------------------------------------
// Exact merge of split units (zwxr.cn 3.3: M = max m_p,
// out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p) and zero output for
// empty sequences.  CTA b >= 1 (hpu warps) owns the unit cut by worker
// boundary b if that is the unit's first interior boundary, one warp per head
// row; CTA 0 zeroes the empty sequences.  Partials are folded in worker order, four segments
// per step (their loads in flight together, M updated once per step).
// ----------------------------------------------------------------------------
template <typename QT, int D, int TT, bool kSuffix>
__global__ void __launch_bounds__(256)
pkv_merge_kernel(const DecodeParams p, int64_t workers, const SuffixArg<kSuffix> sx) {
    // a following programmatic dependent (the cascade's combine pass) may be
    // scheduled now; it waits for this grid before reading
    if constexpr (kSuffix) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t b = blockIdx.x;
    const Lens<kSuffix> ln{p.seq_lens, sx.seq_start, p.num_seqs, p.num_kv_heads * p.nch,
                           p.max_blocks_per_seq * p.block_size};
    if (b == 0) {
        // sequences with nothing to attend: zero output (or an empty partial
        // (m, l) = (-inf, 0) for a cascade suffix); warps scan 32 at a time
        for (int s0 = warp * 32; s0 < p.num_seqs; s0 += blockDim.x) {
            const int sl = s0 + lane;
            unsigned empty = __ballot_sync(kFull, sl < p.num_seqs && ln.eff(sl) == 0);
            while (empty) {
                const int s = s0 + __ffs(empty) - 1;
                empty &= empty - 1;
                if constexpr (kSuffix) {
                    if (ln.first(s) > 0) {
                        for (int i = lane; i < p.num_heads * D; i += 32)
                            sx.part_o[(int64_t)s * p.num_heads * D + i] = 0.f;
                        for (int h = lane; h < p.num_heads; h += 32)
                            sx.part_ml[(int64_t)s * p.num_heads + h] = make_float2(-INFINITY, 0.f);
                        continue;
                    }
                }
                QT* out = reinterpret_cast<QT*>(p.out) + (int64_t)s * p.num_heads * D;
                for (int i = lane; i < p.num_heads * D; i += 32) out[i] = from_f32<QT>(0.f);
            }
        }
        return;
    }
    if (b >= workers) return;
    // every warp locates the boundary's unit itself (no block barrier)
    const int64_t W = total_tiles<TT>(ln);
    const int64_t chunk = (W + workers - 1) / workers;
    const int64_t P = b * chunk;
    if (P >= W) return;
    const SeqHit hit = find_seq<TT>(ln, P);
    const int nt = ntiles_of<TT>(ln.eff_of(hit.L, hit.st));
    const int j = (int)((P - hit.base) / nt);
    const int off = (int)((P - hit.base) % nt);
    const int64_t T0 = hit.base + (int64_t)j * nt;
    if (off == 0 || (b - 1) * chunk > T0) return;   // not an interior first boundary
    const int64_t bf = T0 / chunk, bl = (T0 + nt - 1) / chunk;
    const int kh = j / p.nch, c = j % p.nch;
    const int nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
    const int h = warp;
    if (h >= nh) return;
    // launched as a programmatic dependent of the decode grid: its partials
    // are complete and visible only after this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t u = ((int64_t)hit.s * p.num_kv_heads + kh) * p.nch + c;
    const int64_t row0 = (int64_t)hit.s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c;
    constexpr int PER = D / 32;
    constexpr int kBatch = 4;
    float M = -INFINITY, ls = 0.f, o[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;
    for (int64_t w0 = bf; w0 <= bl; w0 += kBatch) {
        float2 ml[kBatch];
        float v[kBatch][PER];
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const int64_t w = w0 + k;
            ml[k] = make_float2(-INFINITY, 0.f);
#pragma unroll
            for (int e = 0; e < PER; ++e) v[k][e] = 0.f;
            if (w <= bl) {
                ml[k] = p.ws_ml[(w + u) * p.hpu + h];
                const float* src = p.ws_o + ((w + u) * p.hpu + h) * D;
#pragma unroll
                for (int e = 0; e < PER; ++e) v[k][e] = src[lane + 32 * e];
            }
        }
        float Mb = M;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) Mb = fmaxf(Mb, ml[k].x);
        if (Mb == -INFINITY) continue;  // nothing attended yet
        const float fo = M == -INFINITY ? 0.f : ex2(M - Mb);
        ls *= fo;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] *= fo;
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            const float f = ml[k].x == -INFINITY ? 0.f : ex2(ml[k].x - Mb);
            ls += ml[k].y * f;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] += v[k][e] * f;
        }
        M = Mb;
    }
    if constexpr (kSuffix) {
        if (ln.first(hit.s) > 0) {   // cascade suffix: keep the partial
#pragma unroll
            for (int e = 0; e < PER; ++e) sx.part_o[(row0 + h) * D + lane + 32 * e] = o[e];
            if (lane == 0) sx.part_ml[row0 + h] = make_float2(M, ls);
            return;
        }
    }
    QT* out = reinterpret_cast<QT*>(p.out) + (row0 + h) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) out[lane + 32 * e] = from_f32<QT>(ls > 0.f ? o[e] / ls : 0.f);
}


// ----------------------------------------------------------------------------
// The same merge for large batches, where every CTA of the one-boundary form
// would repeat a long length scan: CTA c stands for the 8 worker boundaries
// 8c .. 8c+7 (a warp each) and locates them with one CTA-wide pass over the
// lengths, while the decode grid still runs for the CTAs resident beside it.
// After the decode grid completes, the CTA's warps take the owned units'
// head rows in turn.
// ----------------------------------------------------------------------------
constexpr int kMergeWarps = 8;  // boundaries (and warps) per CTA

struct MergeTask {
    int64_t u;       // unit index (workspace segment base)
    int64_t row0;    // output row of the unit's first head
    int64_t bf, bl;  // first and last worker holding a segment of the unit
    int s;           // its sequence
};

template <typename QT, int D, int TT, bool kSuffix>
__global__ void __launch_bounds__(kMergeWarps * 32)
pkv_merge_wide_kernel(const DecodeParams p, int64_t workers, const SuffixArg<kSuffix> sx) {
    // a following programmatic dependent (the cascade's combine pass) may be
    // scheduled now; it waits for this grid before reading
    if constexpr (kSuffix) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t gw = (int64_t)blockIdx.x * kMergeWarps + warp;
    const Lens<kSuffix> ln{p.seq_lens, sx.seq_start, p.num_seqs, p.num_kv_heads * p.nch,
                           p.max_blocks_per_seq * p.block_size};
    // sequences with nothing to attend (independent of the decode grid): zero
    // output, or an empty partial (m, l) = (-inf, 0) for a cascade suffix; a
    // warp per 32 sequences
    for (int64_t s0 = gw * 32; s0 < p.num_seqs; s0 += (int64_t)gridDim.x * kMergeWarps * 32) {
        const int sl = (int)s0 + lane;
        unsigned empty = __ballot_sync(kFull, sl < p.num_seqs && ln.eff(sl) == 0);
        while (empty) {
            const int s = (int)s0 + __ffs(empty) - 1;
            empty &= empty - 1;
            if constexpr (kSuffix) {
                if (ln.first(s) > 0) {
                    for (int i = lane; i < p.num_heads * D; i += 32)
                        sx.part_o[(int64_t)s * p.num_heads * D + i] = 0.f;
                    for (int h = lane; h < p.num_heads; h += 32)
                        sx.part_ml[(int64_t)s * p.num_heads + h] = make_float2(-INFINITY, 0.f);
                    continue;
                }
            }
            QT* out = reinterpret_cast<QT*>(p.out) + (int64_t)s * p.num_heads * D;
            for (int i = lane; i < p.num_heads * D; i += 32) out[i] = from_f32<QT>(0.f);
        }
    }

    // the CTA's boundaries (every warp takes part in the scans)
    __shared__ BlockScanSmem scan_sm;
    __shared__ MergeTask tasks[kMergeWarps];
    __shared__ int task_nh[kMergeWarps];
    const int64_t W = block_total_tiles<TT>(ln, scan_sm);
    const int64_t chunk = (W + workers - 1) / workers;
    const int64_t b = gw;
    const int64_t P = (b >= 1 && b < workers) ? min(W, b * chunk) : W;
    const SeqHit hit = block_find_seq<TT>(ln, P, scan_sm);
    int nh = 0;
    if (P < W) {
        const int nt = ntiles_of<TT>(ln.eff_of(hit.L, hit.st));
        const int j = (int)((P - hit.base) / nt);
        const int off = (int)((P - hit.base) % nt);
        const int64_t T0 = hit.base + (int64_t)j * nt;
        if (off != 0 && (b - 1) * chunk <= T0) {  // the unit's first interior boundary
            const int kh = j / p.nch, c = j % p.nch;
            nh = min(kHeadsPerUnit, p.g - kHeadsPerUnit * c);
            if (lane == 0) {
                tasks[warp] = MergeTask{((int64_t)hit.s * p.num_kv_heads + kh) * p.nch + c,
                                        (int64_t)hit.s * p.num_heads + (int64_t)kh * p.g + kHeadsPerUnit * c,
                                        T0 / chunk, (T0 + nt - 1) / chunk, hit.s};
            }
        }
    }
    if (lane == 0) task_nh[warp] = nh;
    if (!__syncthreads_or(nh > 0)) return;
    // launched as a programmatic dependent of the decode grid: its partials
    // are complete and visible only after this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int rows = 0;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) rows += task_nh[w];
    constexpr int PER = D / 32;
    constexpr int kBatch = 4;
    for (int q = warp; q < rows; q += kMergeWarps) {
        int tw = 0, h = q;
        while (h >= task_nh[tw]) h -= task_nh[tw++];
        const MergeTask t = tasks[tw];
        float M = -INFINITY, ls = 0.f, o[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] = 0.f;
        for (int64_t w0 = t.bf; w0 <= t.bl; w0 += kBatch) {
            float2 ml[kBatch];
            float v[kBatch][PER];
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int64_t w = w0 + k;
                ml[k] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int e = 0; e < PER; ++e) v[k][e] = 0.f;
                if (w <= t.bl) {
                    ml[k] = p.ws_ml[(w + t.u) * p.hpu + h];
                    const float* src = p.ws_o + ((w + t.u) * p.hpu + h) * D;
#pragma unroll
                    for (int e = 0; e < PER; ++e) v[k][e] = src[lane + 32 * e];
                }
            }
            float Mb = M;
#pragma unroll
            for (int k = 0; k < kBatch; ++k) Mb = fmaxf(Mb, ml[k].x);
            if (Mb == -INFINITY) continue;  // nothing attended yet
            const float fo = M == -INFINITY ? 0.f : ex2(M - Mb);
            ls *= fo;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] *= fo;
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const float f = ml[k].x == -INFINITY ? 0.f : ex2(ml[k].x - Mb);
                ls += ml[k].y * f;
#pragma unroll
                for (int e = 0; e < PER; ++e) o[e] += v[k][e] * f;
            }
            M = Mb;
        }
        if constexpr (kSuffix) {
            if (ln.first(t.s) > 0) {  // cascade suffix: keep the partial
#pragma unroll
                for (int e = 0; e < PER; ++e) sx.part_o[(t.row0 + h) * D + lane + 32 * e] = o[e];
                if (lane == 0) sx.part_ml[t.row0 + h] = make_float2(M, ls);
                continue;
            }
        }
        QT* out = reinterpret_cast<QT*>(p.out) + (t.row0 + h) * D;
#pragma unroll
        for (int e = 0; e < PER; ++e) out[lane + 32 * e] = from_f32<QT>(ls > 0.f ? o[e] / ls : 0.f);
    }
}

}  // namespace pkv
