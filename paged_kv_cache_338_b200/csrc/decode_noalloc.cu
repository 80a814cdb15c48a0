// pa_decode_noalloc: paged decode with a built-in split-K scratch area.
//
// Some callers cannot hand pa_decode a workspace: a serving runtime that
// reserves all device memory for its KV cache up front and owns the only
// allocator; a plugin living inside a host framework that exposes no device
// allocation hook; a latency-bound step loop that may not call cudaMalloc or
// cudaFree (cudaFree waits for the whole device) once it is running.  For
// them this entry point keeps the split-K partials in a fixed, file-scope
// device array instead, and allocates nothing itself.
//
// The array is part of the library's device image: every GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  All calls
// share it, so calls whose device work overlaps (two streams, two host
// threads) race on it and must be serialised by the caller.  Nothing in it has
// to start at zero: every partial the merge reads is written by the same call.
#include <cuda_runtime.h>

#include <mutex>

#include "pa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = PA_DECODE_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array for the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with that device current, and cached per device and context (a
// cudaDeviceReset gives the device a new context, and the next call looks the
// address up again).
void* scratch_address() {
    static pa::SymbolCache cache;
    return pa::symbol_address(g_noalloc_scratch, &cache, "cudaGetSymbolAddress(scratch)");
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, pa_dtype q_dt,
                                       const void* key_cache, const void* value_cache,
                                       pa_dtype cache_dt, const int32_t* block_tables, int MB,
                                       const int32_t* context_lens, int S, int Hq, int Hkv, int D,
                                       int bs, int64_t NB, int max_ctx, float scale,
                                       float k_scale, float v_scale, int partition,
                                       pa_stream_t stream) {
    PA_NVTX_RANGE("pa_decode_noalloc");
    pa::clear_error();
    size_t need = 0;
    pa_status st = pa_decode_workspace_size(S, Hq, D, max_ctx, partition, &need);
    if (st) return st;
    if (need > kNoAllocScratchBytes)
        return pa::fail(PA_ERR_INVALID_ARG,
                        "split-K partials need %zu bytes; the built-in scratch holds %zu "
                        "(use a larger partition, or pa_decode with a workspace)",
                        need, kNoAllocScratchBytes);
    void* ws = nullptr;
    if (need) {
        ws = scratch_address();
        if (!ws) return PA_ERR_CUDA;
    }
    return pa_decode(out, q, q_dt, key_cache, value_cache, cache_dt, block_tables, MB,
                     context_lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale, k_scale, v_scale,
                     partition, ws, need ? kNoAllocScratchBytes : 0, stream);
}
