// noalloc.cu -- pkv_paged_attention_decode_noalloc: the decode attention
// entry point for callers that cannot hand the library a workspace.
//
// The split-merge scratch lives in one file-scope device array of a fixed
// size (kStaticWorkspaceBytes).  Every GPU that loads this library holds it
// until the process exits.  Host code cannot pass the array's name to a
// kernel (on the host it is only a stand-in symbol), so its device address is
// looked up once per device with cudaGetSymbolAddress while that device is
// current, and that address is what the existing decode path receives.
#include <mutex>

#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr size_t kStaticWorkspaceBytes = (size_t)PKV_STATIC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

void* g_ws_ptr[kMaxDevices] = {nullptr};
std::mutex g_ws_mu;

// Device address of the static scratch on the current device (first call on a
// device does the lookup); null on failure.
void* static_workspace(pkv_status* st) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = fail(PKV_ECUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(g_ws_mu);
    if (!g_ws_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_workspace);
        if (e != cudaSuccess || !p) {
            *st = fail(PKV_ECUDA, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
            return nullptr;
        }
        g_ws_ptr[dev] = p;
    }
    return g_ws_ptr[dev];
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_paged_attention_decode_noalloc(
    void* out, const void* query, pkv_dtype q_dtype, const void* key_cache, const void* value_cache,
    pkv_dtype cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
    int block_size, int64_t num_blocks, float scale, const float* k_scale, const float* v_scale,
    int num_ctas, pkv_stream_t stream) {
    if (num_seqs > 0) {
        const size_t need = pkv_paged_attention_workspace_bytes(num_seqs, num_heads, num_kv_heads,
                                                                head_dim, num_ctas);
        if (need > kStaticWorkspaceBytes)
            return fail(PKV_EINVAL,
                        "this call needs %zu bytes of scratch but the static scratch holds %zu "
                        "bytes; use pkv_paged_attention_decode with a caller workspace",
                        need, kStaticWorkspaceBytes);
    }
    pkv_status st = PKV_OK;
    void* ws = static_workspace(&st);
    if (!ws) return st;
    // The existing path, unchanged, with the static array as its workspace.
    // Nothing in it needs zeroing: every partial the merge kernel reads was
    // written earlier in the same call.
    return pkv_paged_attention_decode(out, query, q_dtype, key_cache, value_cache, cache_dtype,
                                      block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                                      num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                                      scale, k_scale, v_scale, ws, kStaticWorkspaceBytes, num_ctas,
                                      stream);
}
