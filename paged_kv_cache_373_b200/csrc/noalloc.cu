// noalloc.cu -- pkv_paged_attention_decode_noalloc: the decode attention
// entry point for callers that cannot hand the library a workspace.
//
// The split-merge scratch lives in one file-scope device array of a fixed
// size (kStaticWorkspaceBytes).  Host code cannot pass the array's name to a
// kernel (on the host it is only a stand-in symbol), so its device address is
// looked up with cudaGetSymbolAddress with the device current and handed to
// the existing decode path.  The address is cached per context (keyed by the
// context's unique id): a call in a context it has not seen before -- another
// device, or the same device after a cudaDeviceReset -- looks it up again, so
// an address never outlives the context it belongs to.
//
// With lazy module loading (the CUDA default, CUDA_MODULE_LOADING=LAZY) the
// array is committed on a device by the first lookup there, i.e. by the first
// call on that device; with eager loading it is committed when the context is
// created.  Either way it stays until the process exits.
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr size_t kStaticWorkspaceBytes = (size_t)PKV_STATIC_WORKSPACE_BYTES;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of the static scratch in the current context; null on failure.
void* static_workspace(pkv_status* st) {
    static SymbolCache cache;
    void* p = symbol_address(g_static_workspace, &cache);
    if (!p) *st = fail(PKV_ECUDA, "cudaGetSymbolAddress(static workspace) failed");
    return p;
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
