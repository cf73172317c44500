/*
 * pkv.h -- C ABI of the B200 (sm_100a) paged KV-cache decode library.
 *
 * The KV cache of one attention layer is a pool of fixed-size physical
 * blocks; each sequence reaches its blocks through a per-sequence block table
 * (zwxr.cn/news/121728 "PagedAttention 与 Continuous Batching", sections 3.1
 * and 3.2).  This library implements the device side of one decode step:
 *
 *   pkv_copy_blocks            copy-on-write copies of shared blocks (3.4)
 *   pkv_swap_blocks            block moves between device and page-locked host
 *                              pools (preemption by swapping, 4.3)
 *   pkv_reshape_and_cache      write each new token's K/V into its slot (3.1)
 *   pkv_paged_attention_decode single-token attention through the block
 *                              table with the block-wise softmax merge (3.3)
 *   pkv_paged_attention_decode_cascade  decode with shared prompt prefixes
 *                              read once per group (3.4)
 *   pkv_paged_prefill          chunked-prefill (causal, multi-token) attention
 *                              through the block table
 * and, in pkv_block_manager.h, the host block manager that produces the
 * tables, slots and copy-on-write pairs.
 *
 * Conventions for every call
 *   - The caller owns all memory.  Pointers named d_* or documented as
 *     "device" are CUDA device pointers; "host" pointers are CPU memory.
 *     The library allocates nothing (its only device state is a static
 *     error word).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) except pkv_get_device_error and pkv_decode_step_host,
 *     which synchronise it.
 *   - Arguments are validated on the host before any launch: a bad argument
 *     returns PKV_EINVAL, a valid but unimplemented combination
 *     PKV_EUNSUPPORTED, and nothing is launched.  A CUDA launch/copy failure
 *     returns PKV_ECUDA.
 *   - Data-dependent faults (a block id outside [0, num_blocks), a slot past
 *     the pool, a seq_len longer than its table row) are detected on the
 *     device: the offending access is skipped or clamped to block 0, the
 *     result is unspecified, and a bit is OR-ed into the device error word
 *     that pkv_get_device_error returns.  Nothing traps.
 *   - Thread safety: calls on different streams may run concurrently; calls
 *     that share a workspace must be ordered by the caller.
 *
 * Layouts (row-major, innermost last):
 *   query, out        [num_seqs, num_heads, head_dim]           q dtype
 *   new key/value     [num_tokens, num_kv_heads, head_dim]      source dtype
 *   key/value cache   [num_blocks, block_size, num_kv_heads, head_dim]
 *   block_tables      int32 [num_seqs, max_blocks_per_seq]
 *   seq_lens          int32 [num_seqs]
 *   slot_mapping      int64 [num_tokens]
 *   block_mapping     int64 [num_pairs, 2]  (src, dst)
 * GQA: q head h reads kv head h / (num_heads / num_kv_heads).
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pkv_stream_t; /* same type as cudaStream_t */

typedef enum {
    PKV_F32 = 0,
    PKV_F16 = 1,
    PKV_BF16 = 2,
    PKV_FP8_E4M3 = 3 /* OCP E4M3 "fn": max 448, no inf, S.1111.111 = NaN */
} pkv_dtype;

typedef enum {
    PKV_OK = 0,
    PKV_EINVAL = 1,       /* bad argument (null pointer, bad shape, bad alignment) */
    PKV_EUNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96) */
    PKV_ECUDA = 3,        /* a CUDA runtime call failed */
    PKV_EDEVICE = 4,      /* the device error word is non-zero */
    PKV_ENOBLOCKS = 5     /* host block manager: the pool cannot supply the blocks */
} pkv_status;

/* Bits of the device error word. */
#define PKV_DEVERR_BLOCK_ID 0x1   /* block table entry outside [0, num_blocks) */
#define PKV_DEVERR_SLOT     0x2   /* slot_mapping entry >= num_blocks * block_size */
#define PKV_DEVERR_SEQ_LEN  0x4   /* seq_len < 0 or > max_blocks_per_seq * block_size */
#define PKV_DEVERR_COPY_ID  0x8   /* copy_blocks src/dst outside [0, num_blocks) */
#define PKV_DEVERR_TIMEOUT  0x10  /* a bounded wait for tensor-core results ran out (pkv_paged_prefill);
                                     the affected rows are not written */

/*
 * pkv_reshape_and_cache -- store the K/V of new tokens in their cache slots.
 * zwxr.cn section 3.1: a token occupies a slot once it is produced; the slot
 * is physical_block * block_size + offset (section 3.2).
 *
 * For i in [0, num_tokens) with s = slot_mapping[i]:
 *   s < 0                     : token i is padding, skipped;
 *   s >= num_blocks*block_size: skipped, PKV_DEVERR_SLOT;
 *   else key_cache[s / block_size, s % block_size, :, :] = key[i, :, :]
 *        (same for value).
 * cache_dtype == src_dtype  : a bit-exact copy (f32, f16 or bf16).
 * cache_dtype == FP8_E4M3   : src_dtype in {f32, f16, bf16}; each element is
 *   stored as round-to-nearest-even, saturating E4M3 of the IEEE fp32
 *   quotient x / *k_scale (resp. *v_scale); NaN stays NaN.  k_scale and
 *   v_scale are device pointers to one fp32 each, required for FP8 and
 *   ignored otherwise.
 * key, value, key_cache, value_cache must be 16-byte aligned.
 * head_dim in {64, 128}; block_size > 0; num_kv_heads > 0.
 */
pkv_status pkv_reshape_and_cache(const void* key, const void* value, pkv_dtype src_dtype,
                                 void* key_cache, void* value_cache, pkv_dtype cache_dtype,
                                 const int64_t* slot_mapping, int64_t num_tokens,
                                 int64_t num_blocks, int block_size, int num_kv_heads,
                                 int head_dim, const float* k_scale, const float* v_scale,
                                 pkv_stream_t stream);

/*
 * pkv_copy_blocks -- copy-on-write duplication of whole physical blocks.
 * zwxr.cn section 3.4 / ttlab.hopto.org section 2: shared blocks are
 * read-only; a sequence about to write into a shared block first copies it.
 *
 * For every pair p and every layer l:
 *   key_caches[l] block block_mapping[p][1] = key_caches[l] block block_mapping[p][0]
 * (same for value_caches), each block being block_bytes contiguous bytes
 * (block_size * num_kv_heads * head_dim * element size), unused slots included.
 * key_caches / value_caches: HOST arrays of num_layers DEVICE pointers
 * (num_layers in [1, 128]); block_mapping: DEVICE int64 [num_pairs, 2].
 * block_bytes must be a multiple of 16 and every cache 16-byte aligned.
 * Destinations must be distinct and disjoint from all sources (otherwise
 * the result is unspecified).  Ids outside [0, num_blocks) skip the pair
 * and set PKV_DEVERR_COPY_ID.
 */
pkv_status pkv_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                           const int64_t* block_mapping, int64_t num_pairs, int64_t num_blocks,
                           size_t block_bytes, pkv_stream_t stream);

/*
 * pkv_swap_blocks -- whole-block copies from one block pool to another, where
 * each pool lives in device memory of the current device or in page-locked
 * host memory (cudaHostAlloc / cudaHostRegister, torch pin_memory), which the
 * kernel reads and writes directly through unified addressing.  This is the
 * data movement of preemption by swapping (zwxr.cn section 4.3): the blocks
 * of a preempted sequence go to host memory, and later come back to whatever
 * device blocks are free (its block table is rewritten by the caller).
 *
 * For every pair p and every layer l:
 *   dst_key_caches[l] block block_mapping[p][1] = src_key_caches[l] block block_mapping[p][0]
 * (same for values); blocks are block_bytes contiguous bytes (a multiple of
 * 16), pools 16-byte aligned.  dst/src_*_caches: HOST arrays of num_layers
 * pool pointers (num_layers in [1, 128]); block_mapping: int64 [num_pairs, 2]
 * in device or page-locked host memory.  A source id outside
 * [0, src_num_blocks) or destination id outside [0, dst_num_blocks) skips the
 * pair and sets PKV_DEVERR_COPY_ID.  Destinations must be distinct and must
 * not overlap a source block (otherwise the result is unspecified).
 * Returns PKV_EINVAL for pageable host memory or a pointer CUDA does not
 * know, and PKV_EUNSUPPORTED for memory of another device; the caller keeps
 * host pools alive and unmodified until the stream has passed the copy.
 */
pkv_status pkv_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                           int64_t dst_num_blocks, const void* const* src_key_caches,
                           const void* const* src_value_caches, int64_t src_num_blocks,
                           int num_layers, const int64_t* block_mapping, int64_t num_pairs,
                           size_t block_bytes, pkv_stream_t stream);

/*
 * Workspace for pkv_paged_attention_decode: fp32 partial results of the
 * split units, (12 * num_ctas + units) x heads_per_unit x (head_dim + 2)
 * floats, where units = num_seqs * num_kv_heads * ceil(g / 8),
 * g = num_heads / num_kv_heads and heads_per_unit = min(g, 8).  num_ctas = 0 means the default grid of the
 * current device (pkv_default_num_ctas).  Returns 0 for invalid shapes
 * (num_ctas outside [0, 2^20] included).
 * The workspace needs no initialisation.
 */
size_t pkv_paged_attention_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                           int head_dim, int num_ctas);

/* Persistent grid size used when num_ctas = 0: one CTA per SM of the
 * current device (148 on B200).  Returns 0 on error. */
int pkv_default_num_ctas(void);

/*
 * pkv_paged_attention_decode -- single-token decode attention over a paged
 * KV cache.  thinkmoon.cn "PagedAttention不够用了之后" (the paged_attention
 * pseudocode: gather the sequence's blocks, q.K^T / sqrt(d), softmax, .V)
 * with zwxr.cn section 3.3 (block-wise softmax: per-block running max m and
 * normaliser l merged by rescaling, exactly the global softmax).
 *
 * For every sequence s (L = seq_lens[s]) and q head h (kv head kh = h / g):
 *   score_t = scale * <query[s,h,:], K_t>       for t in [0, L)
 *   out[s,h,:] = sum_t softmax(score)_t * V_t   (L == 0 -> zeros)
 * where K_t / V_t is row (block_tables[s][t / block_size], t % block_size, kh)
 * of the caches (times *k_scale / *v_scale for FP8 caches).
 *
 * Supported: cache_dtype f32 (q f32), f16 (q f16), bf16 (q bf16),
 *   FP8_E4M3 (q f16 or bf16, head_dim 128); head_dim in {64, 128};
 *   block_size in {16, 32}; num_heads % num_kv_heads == 0; any g.
 * Numerics: fp32 accumulation and fp32 online softmax; for 16-bit and FP8
 * caches the q.K and P.V products run on tensor cores with 16-bit operands
 * (P rounded to the cache's 16-bit type, f16 for FP8).  Output is rounded
 * to the q dtype (RNE).
 * Every warp of the persistent grid takes an equal share of all
 * (sequence, kv head) tiles, so long sequences are split across warps and
 * their partial (m, l, o) are merged exactly by a second kernel on the same
 * stream.  Results are bit-identical under any permutation of the
 * physical block ids and independent of block sharing, for a fixed num_ctas.
 * workspace: device, >= pkv_paged_attention_workspace_bytes(...) bytes,
 *   16-byte aligned, contents need no initialisation.
 * num_ctas: 0 = default; otherwise the persistent grid size (sets the split),
 *   at most 2^20 (PKV_EINVAL above).
 * out, query, caches: 16-byte aligned device pointers.
 */
pkv_status pkv_paged_attention_decode(void* out, const void* query, pkv_dtype q_dtype,
                                      const void* key_cache, const void* value_cache,
                                      pkv_dtype cache_dtype, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* seq_lens,
                                      int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int block_size, int64_t num_blocks,
                                      float scale, const float* k_scale, const float* v_scale,
                                      void* workspace, size_t workspace_bytes, int num_ctas,
                                      pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_cascade -- decode attention for batches in which
 * groups of sequences share a prompt prefix through shared physical blocks
 * (copy-on-write sharing: zwxr.cn section 3.4; ttlab.hopto.org section 2,
 * parallel sampling and beam search).  The shared prefix blocks of a group are
 * read from memory once per kv head for all members, instead of once per
 * member; the result is the same attention as pkv_paged_attention_decode
 * (prefix and suffix are two partial softmaxes merged exactly with the
 * block-wise (m, l) rule of zwxr.cn section 3.3).
 *
 * Groups (all DEVICE int32 arrays):
 *   group_offsets [num_groups + 1]  CSR offsets; group i's members are
 *                                   group_members[group_offsets[i] .. group_offsets[i+1])
 *   group_members                   sequence ids; a sequence in at most one group
 *   group_prefix_lens [num_groups]  requested shared prefix length (tokens)
 *   max_group_size                  upper bound on members per group (host)
 * The prefix actually shared by group i is computed on the device: the
 * longest run of leading table entries that all members have in common,
 * capped by group_prefix_lens[i] and by every member's length, in whole
 * blocks (a request longer than a member's length sets PKV_DEVERR_SEQ_LEN, as
 * does a group with more than max_group_size members, which is then not
 * shared).  A shared run shorter than 32 tokens is not worth a separate pass:
 * such a group is decoded unshared.  group_offsets must be a valid
 * non-decreasing CSR index.
 * Sequences outside every group, groups of one member and cache dtypes other
 * than f16/bf16 take the ordinary decode path.
 * workspace: >= pkv_paged_attention_cascade_workspace_bytes(...) bytes, no
 * initialisation needed.  Other arguments as pkv_paged_attention_decode.
 */
size_t pkv_paged_attention_cascade_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                                   int head_dim, int num_groups,
                                                   int max_group_size, int num_ctas);

pkv_status pkv_paged_attention_decode_cascade(void* out, const void* query, pkv_dtype q_dtype,
                                              const void* key_cache, const void* value_cache,
                                              pkv_dtype cache_dtype, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* seq_lens,
                                              int num_seqs, const int32_t* group_offsets,
                                              const int32_t* group_members,
                                              const int32_t* group_prefix_lens, int num_groups,
                                              int max_group_size, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size, int64_t num_blocks,
                                              float scale, const float* k_scale,
                                              const float* v_scale, void* workspace,
                                              size_t workspace_bytes, int num_ctas,
                                              pkv_stream_t stream);

/*
 * pkv_paged_prefill -- chunked-prefill attention over the paged cache
 * (ttlab.hopto.org "LLM KV cache 02", section 3: a long prompt is cut into
 * chunks that share each step's token budget with decode tokens).
 *
 * Sequence s contributes the chunk rows query[query_start[s] .. query_start[s+1])
 * (C_s = query_start[s+1] - query_start[s] tokens; C_s = 1 is a decode row).
 * The cache already holds all seq_lens[s] tokens of the sequence, the
 * chunk's own K/V included (pkv_reshape_and_cache first), so chunk token i is
 * at position p = seq_lens[s] - C_s + i and
 *   out[query_start[s] + i, h, :] = softmax_t<=p(scale * q . K[t, h / g]) . V
 * (causal attention through the block table; g = num_heads / num_kv_heads).
 * query, out: [num_query_tokens, num_heads, head_dim] (device, 16-byte
 * aligned); query_start: DEVICE int32 [num_seqs + 1], non-decreasing, with
 * query_start[num_seqs] == num_query_tokens (host-known, sizes the grid);
 * caches, tables, seq_lens as pkv_paged_attention_decode.
 * Supported: f16 or bf16 caches with q and out of the same dtype,
 * head_dim in {64, 128}, block_size in {16, 32}, g in {1, 2, 4, 8, 16}
 * (otherwise PKV_EUNSUPPORTED).  A seq_len shorter than its chunk or longer
 * than its table row, or a decreasing query_start, sets PKV_DEVERR_SEQ_LEN
 * (those rows are not written); an out-of-range block id is read as block 0
 * (the affected rows are unspecified) and sets PKV_DEVERR_BLOCK_ID.
 * num_query_tokens and num_blocks * block_size must stay below 2^31 (32-bit
 * copy coordinates; otherwise PKV_EUNSUPPORTED).  No workspace.  The
 * products run on the tensor core with accumulators in tensor memory: one
 * CTA per SM holding all 512 columns; q and K/V tiles are copied by TMA.
 */
pkv_status pkv_paged_prefill(void* out, const void* query, pkv_dtype q_dtype, const void* key_cache,
                             const void* value_cache, pkv_dtype cache_dtype,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* seq_lens, const int32_t* query_start, int num_seqs,
                             int64_t num_query_tokens, int num_heads, int num_kv_heads, int head_dim,
                             int block_size, int64_t num_blocks, float scale, pkv_stream_t stream);

/* Size of the static scratch used by pkv_paged_attention_decode_noalloc. */
#define PKV_STATIC_WORKSPACE_BYTES (16u * 1024u * 1024u)

/*
 * pkv_paged_attention_decode_noalloc -- pkv_paged_attention_decode with no
 * workspace argument.  The pages have no counterpart: this entry point is for
 * callers that cannot allocate device memory at the point where they decode,
 * e.g. a serving engine that reserved (nearly) all device memory for its KV
 * block pool before the first step, a plugin that has no access to its host
 * framework's allocator, or a latency-critical decode loop where cudaMalloc /
 * cudaFree would synchronise the device and stall every other stream.
 *
 * Same arguments, semantics and results as pkv_paged_attention_decode; the
 * split-merge scratch is one file-scope device array of
 * PKV_STATIC_WORKSPACE_BYTES (16 MiB), held on a device until the process
 * exits.  The call itself runs no cudaMalloc, cudaFree or allocating library
 * routine.
 *   - Limit: if pkv_paged_attention_workspace_bytes(num_seqs, num_heads,
 *     num_kv_heads, head_dim, num_ctas) exceeds PKV_STATIC_WORKSPACE_BYTES the
 *     call returns PKV_EINVAL and launches nothing.
 *   - Set-up: the array's device address is looked up (cudaGetSymbolAddress)
 *     by the first call in each CUDA context and cached per context.  Under
 *     lazy module loading (the CUDA default) that first lookup is what commits
 *     the 16 MiB on the device, so the FIRST call on each device may allocate
 *     and synchronise.  Make one warm-up call per device, with that device
 *     current, before the KV pool takes the device memory and before any
 *     stream capture: a call with num_seqs = 0 (dtypes, head_dim, block_size,
 *     num_blocks and max_blocks_per_seq valid; pointers may be NULL) does only
 *     that set-up and returns PKV_OK.  Later calls allocate nothing.  A call
 *     after cudaDeviceReset runs in a new context: it looks the address up
 *     again (and is again a first call).
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     last call's contents.  Nothing in it has to start at zero (every value
 *     read is written earlier by the same call), but calls that overlap on the
 *     GPU (different streams, or threads that do not order their calls) race
 *     on it and give wrong results: order them.
 */
pkv_status pkv_paged_attention_decode_noalloc(void* out, const void* query, pkv_dtype q_dtype,
                                              const void* key_cache, const void* value_cache,
                                              pkv_dtype cache_dtype, const int32_t* block_tables,
                                              int max_blocks_per_seq, const int32_t* seq_lens,
                                              int num_seqs, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size, int64_t num_blocks,
                                              float scale, const float* k_scale,
                                              const float* v_scale, int num_ctas,
                                              pkv_stream_t stream);

/*
 * pkv_decode_step_host -- one whole decode step driven from host buffers:
 * copies the step's inputs host -> device, runs copy_blocks (if
 * num_cow_pairs > 0), reshape_and_cache of one new token per sequence and
 * the decode attention, copies the output device -> host and waits for the
 * stream (the calling thread polls cudaStreamQuery until the step is done,
 * rather than sleeping in cudaStreamSynchronize).  Host buffers should be
 * pinned for asynchronous copies.
 * The caches stay resident on the device.  Device staging buffers are
 * caller-owned and sized like their host counterparts.
 *
 * Packed inputs (h_packed != NULL): the caller writes all the step's inputs
 * into ONE pinned host buffer at the offsets pkv_decode_step_layout gives,
 * and the step moves them with one host -> device copy into d_packed (device,
 * layout.total bytes, 16-byte aligned) instead of one copy per input; the
 * h_query ... h_cow_pairs and d_query ... d_cow_pairs fields are then
 * ignored.  The output still goes d_out -> h_out in one copy.
 */
typedef struct pkv_decode_step_args {
    /* shapes */
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
    int64_t num_blocks;
    pkv_dtype q_dtype;      /* also the dtype of the new K/V rows */
    pkv_dtype cache_dtype;
    float scale;
    int num_ctas;           /* 0 = default */
    /* host inputs / output */
    const void* h_query;              /* [S, Hq, D] */
    const void* h_new_key;            /* [S, Hkv, D] */
    const void* h_new_value;          /* [S, Hkv, D] */
    const int64_t* h_slot_mapping;    /* [S] */
    const int32_t* h_block_tables;    /* [S, max_blocks_per_seq] */
    const int32_t* h_seq_lens;        /* [S] */
    const int64_t* h_cow_pairs;       /* [num_cow_pairs, 2] or NULL */
    int64_t num_cow_pairs;
    void* h_out;                      /* [S, Hq, D] */
    /* device staging (same sizes as the host buffers) */
    void* d_query;
    void* d_new_key;
    void* d_new_value;
    int64_t* d_slot_mapping;
    int32_t* d_block_tables;
    int32_t* d_seq_lens;
    int64_t* d_cow_pairs;
    void* d_out;
    /* device state */
    void* key_cache;
    void* value_cache;
    const float* k_scale;             /* device, FP8 only */
    const float* v_scale;
    void* workspace;
    size_t workspace_bytes;
    /* packed inputs (optional; see above) */
    const void* h_packed;             /* pinned host, layout.total bytes, or NULL */
    void* d_packed;                   /* device, layout.total bytes */
} pkv_decode_step_args;

pkv_status pkv_decode_step_host(const pkv_decode_step_args* args, pkv_stream_t stream);

/* Byte offsets of a decode step's inputs inside one packed buffer: each
 * array starts on a 256-byte boundary, in the order query [S, Hq, D],
 * new_key and new_value [S, Hkv, D] (q dtype), slot_mapping int64 [S],
 * block_tables int32 [S, max_blocks_per_seq], seq_lens int32 [S],
 * cow_pairs int64 [num_cow_pairs, 2]; total = the packed size in bytes. */
typedef struct pkv_step_layout {
    size_t query, new_key, new_value, slot_mapping, block_tables, seq_lens, cow_pairs;
    size_t total;
} pkv_step_layout;

/* Fill *layout for these shapes.  PKV_EINVAL for negative sizes, a bad dtype
 * or a null layout. */
pkv_status pkv_decode_step_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                  pkv_dtype q_dtype, int max_blocks_per_seq,
                                  int64_t num_cow_pairs, pkv_step_layout* layout);

/* Synchronise `stream`, return the device error word of the current device
 * in *code_out and clear it.  Returns PKV_EDEVICE if it was non-zero. */
pkv_status pkv_get_device_error(int32_t* code_out, pkv_stream_t stream);

/* Static description of a status code. */
const char* pkv_status_string(pkv_status status);

/* Detail of the last host-side failure on the calling thread ("" if none). */
const char* pkv_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
