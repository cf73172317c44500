// pkv_api.cu -- host side of pkv_paged_attention_decode and the library
// utilities: argument validation, variant dispatch, workspace layout, the
// device error word and the host-buffer decode step.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <utility>

#include <cudaTypedefs.h>

#include "paged_attention.cuh"
#include "pkv_internal.h"

namespace pkv {

// The library's only device state: OR of PKV_DEVERR_* bits, one per device.
__device__ int g_pkv_error;

namespace {
thread_local char g_msg[512] = "";
}  // namespace

pkv_status fail(pkv_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return st;
}

int dtype_bytes(pkv_dtype d) {
    switch (d) {
    case PKV_F32: return 4;
    case PKV_F16: case PKV_BF16: return 2;
    case PKV_FP8_E4M3: return 1;
    default: return 0;
    }
}

namespace {

// The current context's unique id (cuCtxGetId, through the runtime's driver
// entry points); 0 if there is none or the driver cannot tell.
unsigned long long current_context_id() {
    static const auto fns = [] {
        void* get_current = nullptr;
        void* get_id = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &get_current, 4000, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess)
            get_current = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &get_id, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            get_id = nullptr;
        return std::make_pair(reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(get_current),
                              reinterpret_cast<PFN_cuCtxGetId_v12000>(get_id));
    }();
    if (!fns.first || !fns.second) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (fns.first(&ctx) != CUDA_SUCCESS || !ctx || fns.second(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace

void* symbol_address(const void* symbol, SymbolCache* cache) {
    // the lookup is repeated whenever the current context is not the one the
    // cached address belongs to (another device, or the same device after a
    // reset), so an address never outlives its context
    const unsigned long long ctx = current_context_id();
    if (ctx != 0) {
        std::lock_guard<std::mutex> lk(cache->mu);
        for (const auto& e : cache->entries)
            if (e.first == ctx) return e.second;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return nullptr;
    const unsigned long long ctx2 = ctx != 0 ? ctx : current_context_id();  // the lookup may create it
    if (ctx2 != 0) {
        std::lock_guard<std::mutex> lk(cache->mu);
        if (cache->entries.size() >= 64) cache->entries.erase(cache->entries.begin());
        cache->entries.emplace_back(ctx2, p);
    }
    return p;
}

int* device_error_word() {
    static SymbolCache cache;
    return static_cast<int*>(symbol_address(&g_pkv_error, &cache));
}

static int default_ctas() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

struct WsLayout {
    size_t o_bytes, ml_off, total;
    int hpu, nch, grid;
};

static bool ws_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int num_ctas,
                      WsLayout* w) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return false;
    if (head_dim <= 0 || num_ctas < 0 || num_ctas > kMaxCtas) return false;
    const int g = num_heads / num_kv_heads;
    w->grid = num_ctas > 0 ? num_ctas : default_ctas();
    if (w->grid <= 0) return false;
    w->nch = (g + kHeadsPerUnit - 1) / kHeadsPerUnit;
    w->hpu = g < kHeadsPerUnit ? g : kHeadsPerUnit;
    // one segment per worker (up to kMaxWarpsPerCta warps per CTA) plus one per unit
    const size_t segs = (size_t)w->grid * kMaxWarpsPerCta + (size_t)num_seqs * num_kv_heads * w->nch;
    w->o_bytes = segs * w->hpu * head_dim * sizeof(float);
    w->ml_off = (w->o_bytes + 255) & ~(size_t)255;
    w->total = w->ml_off + segs * w->hpu * sizeof(float2);
    return true;
}

}  // namespace pkv

using namespace pkv;

extern "C" int pkv_default_num_ctas(void) { return default_ctas(); }

extern "C" size_t pkv_paged_attention_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads,
                                                      int head_dim, int num_ctas) {
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, num_ctas, &w)) return 0;
    return w.total;
}

namespace pkv {

pkv_status decode_prepare(DecodeParams* pp, DecodeLauncher* launch_out, int* grid_out, void* out,
                          const void* query, pkv_dtype q_dtype, const void* key_cache,
                          const void* value_cache, pkv_dtype cache_dtype, const int32_t* block_tables,
                          int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, float scale,
                          const float* k_scale, const float* v_scale, void* workspace,
                          size_t workspace_bytes, int num_ctas) {
    *launch_out = nullptr;
    if (num_seqs < 0) return fail(PKV_EINVAL, "num_seqs < 0");
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0)
        return fail(PKV_EINVAL, "num_heads must be a positive multiple of num_kv_heads");
    if (head_dim != 64 && head_dim != 128) return fail(PKV_EUNSUPPORTED, "head_dim %d", head_dim);
    if (block_size != 16 && block_size != 32) return fail(PKV_EUNSUPPORTED, "block_size %d", block_size);
    if (num_blocks <= 0 || num_blocks > 0x7fffffffLL) return fail(PKV_EINVAL, "num_blocks out of range");
    if (max_blocks_per_seq <= 0 || (int64_t)max_blocks_per_seq * block_size > 0x7fffffffLL)
        return fail(PKV_EINVAL, "max_blocks_per_seq out of range");
    if (!std::isfinite(scale)) return fail(PKV_EINVAL, "scale must be finite");
    if (num_ctas < 0 || num_ctas > kMaxCtas) return fail(PKV_EINVAL, "num_ctas %d outside [0, %d]", num_ctas, kMaxCtas);
    // dtype combination -> launcher
    DecodeLauncher launch = nullptr;
    if (cache_dtype == PKV_F32 && q_dtype == PKV_F32)
        launch = head_dim == 64 ? launch_decode_f32_d64 : launch_decode_f32_d128;
    else if (cache_dtype == PKV_F16 && q_dtype == PKV_F16)
        launch = head_dim == 64 ? launch_decode_f16_d64 : launch_decode_f16_d128;
    else if (cache_dtype == PKV_BF16 && q_dtype == PKV_BF16)
        launch = head_dim == 64 ? launch_decode_bf16_d64 : launch_decode_bf16_d128;
    else if (cache_dtype == PKV_FP8_E4M3 && head_dim == 128 && (q_dtype == PKV_F16 || q_dtype == PKV_BF16))
        launch = q_dtype == PKV_F16 ? launch_decode_fp8_qf16_d128 : launch_decode_fp8_qbf16_d128;
    if (!launch) return fail(PKV_EUNSUPPORTED, "q dtype %d with cache dtype %d, head_dim %d",
                             (int)q_dtype, (int)cache_dtype, head_dim);
    if (cache_dtype == PKV_FP8_E4M3 && (!k_scale || !v_scale))
        return fail(PKV_EINVAL, "FP8 cache needs k_scale and v_scale");
    if (num_seqs == 0) return PKV_OK;  // nothing to launch
    if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !workspace)
        return fail(PKV_EINVAL, "null pointer");
    if (!aligned16(out) || !aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache) ||
        !aligned16(workspace))
        return fail(PKV_EINVAL, "out, query, caches and workspace must be 16-byte aligned");
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, num_ctas, &w))
        return fail(PKV_ECUDA, "cannot size the grid");
    if (workspace_bytes < w.total)
        return fail(PKV_EINVAL, "workspace too small: %zu < %zu bytes", workspace_bytes, w.total);
    int* err = device_error_word();
    if (!err) return fail(PKV_ECUDA, "device error word unavailable");

    DecodeParams p{};
    p.out = out;
    p.q = query;
    p.key_cache = static_cast<const uint8_t*>(key_cache);
    p.value_cache = static_cast<const uint8_t*>(value_cache);
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.k_scale = cache_dtype == PKV_FP8_E4M3 ? k_scale : nullptr;
    p.v_scale = cache_dtype == PKV_FP8_E4M3 ? v_scale : nullptr;
    p.ws_o = static_cast<float*>(workspace);
    p.ws_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + w.ml_off);
    p.err = err;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.g = num_heads / num_kv_heads;
    p.nch = w.nch;
    p.hpu = w.hpu;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.block_size = block_size;
    p.num_blocks = (int)num_blocks;
    p.scale_log2 = (float)((double)scale * 1.4426950408889634);
    *pp = p;
    *launch_out = launch;
    *grid_out = w.grid;
    return PKV_OK;
}

size_t decode_workspace_bytes(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int num_ctas) {
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, num_ctas, &w)) return 0;
    return w.total;
}

}  // namespace pkv

extern "C" pkv_status pkv_paged_attention_decode(void* out, const void* query, pkv_dtype q_dtype,
                                                 const void* key_cache, const void* value_cache,
                                                 pkv_dtype cache_dtype, const int32_t* block_tables,
                                                 int max_blocks_per_seq, const int32_t* seq_lens,
                                                 int num_seqs, int num_heads, int num_kv_heads,
                                                 int head_dim, int block_size, int64_t num_blocks,
                                                 float scale, const float* k_scale, const float* v_scale,
                                                 void* workspace, size_t workspace_bytes, int num_ctas,
                                                 pkv_stream_t stream) {
    DecodeParams p;
    DecodeLauncher launch;
    int grid = 0;
    const pkv_status st = decode_prepare(&p, &launch, &grid, out, query, q_dtype, key_cache, value_cache,
                                         cache_dtype, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                         num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                                         k_scale, v_scale, workspace, workspace_bytes, num_ctas);
    if (st != PKV_OK || num_seqs == 0) return st;
    DecodeLaunchArgs a{&p, grid};
    return launch(a, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" pkv_status pkv_decode_step_layout(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                             pkv_dtype q_dtype, int max_blocks_per_seq,
                                             int64_t num_cow_pairs, pkv_step_layout* l) {
    if (!l) return fail(PKV_EINVAL, "null layout");
    const int qb = dtype_bytes(q_dtype);
    if (qb == 0) return fail(PKV_EINVAL, "q dtype");
    if (num_seqs < 0 || num_heads < 0 || num_kv_heads < 0 || head_dim < 0 || max_blocks_per_seq < 0 ||
        num_cow_pairs < 0)
        return fail(PKV_EINVAL, "negative size");
    const size_t S = (size_t)num_seqs;
    size_t at = 0;
    auto take = [&](size_t n) {
        const size_t off = at;
        at = (at + n + 255) & ~(size_t)255;
        return off;
    };
    l->query = take(S * num_heads * head_dim * qb);
    l->new_key = take(S * num_kv_heads * head_dim * qb);
    l->new_value = take(S * num_kv_heads * head_dim * qb);
    l->slot_mapping = take(S * sizeof(int64_t));
    l->block_tables = take(S * max_blocks_per_seq * sizeof(int32_t));
    l->seq_lens = take(S * sizeof(int32_t));
    l->cow_pairs = take((size_t)num_cow_pairs * 2 * sizeof(int64_t));
    l->total = at;
    return PKV_OK;
}

extern "C" pkv_status pkv_decode_step_host(const pkv_decode_step_args* a, pkv_stream_t stream) {
    if (!a) return fail(PKV_EINVAL, "null args");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int S = a->num_seqs;
    if (S < 0) return fail(PKV_EINVAL, "num_seqs < 0");
    const int qb = dtype_bytes(a->q_dtype);
    if (qb == 0) return fail(PKV_EINVAL, "q dtype");
    const size_t q_bytes = (size_t)S * a->num_heads * a->head_dim * qb;
    const size_t kv_bytes = (size_t)S * a->num_kv_heads * a->head_dim * qb;
    const int64_t npairs = a->num_cow_pairs > 0 ? a->num_cow_pairs : 0;
    // device addresses of the step's inputs
    const void* d_query = a->d_query;
    const void* d_new_key = a->d_new_key;
    const void* d_new_value = a->d_new_value;
    const int64_t* d_slots = a->d_slot_mapping;
    const int32_t* d_tables = a->d_block_tables;
    const int32_t* d_lens = a->d_seq_lens;
    const int64_t* d_pairs = a->d_cow_pairs;
    if (a->h_packed) {
        // one copy of the whole packed input buffer
        pkv_step_layout l;
        pkv_status s = pkv_decode_step_layout(S, a->num_heads, a->num_kv_heads, a->head_dim, a->q_dtype,
                                              a->max_blocks_per_seq, npairs, &l);
        if (s != PKV_OK) return s;
        if (!a->d_packed || !aligned16(a->d_packed)) return fail(PKV_EINVAL, "d_packed null or not 16-byte aligned");
        uint8_t* d = static_cast<uint8_t*>(a->d_packed);
        if (l.total) {
            const cudaError_t e = cudaMemcpyAsync(d, a->h_packed, l.total, cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess) return fail(PKV_ECUDA, "H2D copy: %s", cudaGetErrorString(e));
        }
        d_query = d + l.query;
        d_new_key = d + l.new_key;
        d_new_value = d + l.new_value;
        d_slots = reinterpret_cast<const int64_t*>(d + l.slot_mapping);
        d_tables = reinterpret_cast<const int32_t*>(d + l.block_tables);
        d_lens = reinterpret_cast<const int32_t*>(d + l.seq_lens);
        d_pairs = reinterpret_cast<const int64_t*>(d + l.cow_pairs);
    } else {
        struct Cp { const void* dst; const void* src; size_t n; };
        const Cp h2d[] = {
            {a->d_query, a->h_query, q_bytes},
            {a->d_new_key, a->h_new_key, kv_bytes},
            {a->d_new_value, a->h_new_value, kv_bytes},
            {a->d_slot_mapping, a->h_slot_mapping, (size_t)S * sizeof(int64_t)},
            {a->d_block_tables, a->h_block_tables, (size_t)S * a->max_blocks_per_seq * sizeof(int32_t)},
            {a->d_seq_lens, a->h_seq_lens, (size_t)S * sizeof(int32_t)},
            {a->d_cow_pairs, a->h_cow_pairs, (size_t)npairs * 2 * sizeof(int64_t)},
        };
        for (const Cp& c : h2d) {
            if (c.n == 0) continue;
            if (!c.dst || !c.src) return fail(PKV_EINVAL, "null staging or host buffer");
            const cudaError_t e = cudaMemcpyAsync(const_cast<void*>(c.dst), c.src, c.n, cudaMemcpyHostToDevice, st);
            if (e != cudaSuccess) return fail(PKV_ECUDA, "H2D copy: %s", cudaGetErrorString(e));
        }
    }
    pkv_status s;
    if (npairs > 0) {
        void* kcs[1] = {a->key_cache};
        void* vcs[1] = {a->value_cache};
        const size_t block_bytes = (size_t)a->block_size * a->num_kv_heads * a->head_dim *
                                   dtype_bytes(a->cache_dtype);
        if ((s = pkv_copy_blocks(kcs, vcs, 1, d_pairs, npairs, a->num_blocks, block_bytes, stream)) != PKV_OK)
            return s;
    }
    if ((s = pkv_reshape_and_cache(d_new_key, d_new_value, a->q_dtype, a->key_cache, a->value_cache,
                                   a->cache_dtype, d_slots, S, a->num_blocks, a->block_size,
                                   a->num_kv_heads, a->head_dim, a->k_scale, a->v_scale, stream)) != PKV_OK)
        return s;
    if ((s = pkv_paged_attention_decode(a->d_out, d_query, a->q_dtype, a->key_cache, a->value_cache,
                                        a->cache_dtype, d_tables, a->max_blocks_per_seq, d_lens, S,
                                        a->num_heads, a->num_kv_heads, a->head_dim, a->block_size,
                                        a->num_blocks, a->scale, a->k_scale, a->v_scale, a->workspace,
                                        a->workspace_bytes, a->num_ctas, stream)) != PKV_OK)
        return s;
    if (q_bytes) {
        if (!a->h_out || !a->d_out) return fail(PKV_EINVAL, "null output buffer");
        const cudaError_t e = cudaMemcpyAsync(a->h_out, a->d_out, q_bytes, cudaMemcpyDeviceToHost, st);
        if (e != cudaSuccess) return fail(PKV_ECUDA, "D2H copy: %s", cudaGetErrorString(e));
    }
    // wait by polling: the calling thread spins on the stream instead of
    // sleeping in cudaStreamSynchronize, whose wake-up under a context's
    // default scheduling added 10-40 us to a step of a few hundred us
    cudaError_t e;
    while ((e = cudaStreamQuery(st)) == cudaErrorNotReady) {}
    if (e != cudaSuccess) return fail(PKV_ECUDA, "decode step: %s", cudaGetErrorString(e));
    return PKV_OK;
}

extern "C" pkv_status pkv_get_device_error(int32_t* code_out, pkv_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_pkv_error, sizeof(v));
    if (e == cudaSuccess) {
        const int32_t zero = 0;
        e = cudaMemcpyToSymbol(g_pkv_error, &zero, sizeof(zero));
    }
    if (e != cudaSuccess) return fail(PKV_ECUDA, "get_device_error: %s", cudaGetErrorString(e));
    if (code_out) *code_out = v;
    return v ? PKV_EDEVICE : PKV_OK;
}

extern "C" const char* pkv_status_string(pkv_status s) {
    switch (s) {
    case PKV_OK: return "ok";
    case PKV_EINVAL: return "invalid argument";
    case PKV_EUNSUPPORTED: return "unsupported combination";
    case PKV_ECUDA: return "CUDA error";
    case PKV_EDEVICE: return "device-side error flag set";
    case PKV_ENOBLOCKS: return "out of free blocks";
    default: return "unknown status";
    }
}

extern "C" const char* pkv_last_error_message(void) { return g_msg; }
