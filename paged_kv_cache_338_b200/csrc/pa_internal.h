// Host-side internals shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>

#include <vector_types.h>

#include "pa.h"

// Profiler ranges around the C-ABI entry points (a named NVTX range per call,
// seen on an Nsight Systems timeline).  Compiled in only when the library is
// built with PA_WITH_NVTX (python -m paged_kv_cache_338_b200.build --nvtx);
// otherwise the macro is empty and costs nothing.
#ifdef PA_WITH_NVTX
#include <nvtx3/nvToolsExt.h>
namespace pa {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace pa
#define PA_NVTX_RANGE(name) ::pa::NvtxRange pa_nvtx_range_(name)
#else
#define PA_NVTX_RANGE(name) ((void)0)
#endif

namespace pa {

// Record a failure for pa_last_error() on this thread and return the status.
pa_status fail(pa_status st, const char* fmt, ...);
void clear_error();

inline int elem_size(pa_dtype dt) {
    switch (dt) {
    case PA_F32: return 4;
    case PA_F16: case PA_BF16: return 2;
    case PA_FP8_E4M3: return 1;
    }
    return 0;
}

inline bool valid_dtype(int dt) { return dt >= PA_F32 && dt <= PA_FP8_E4M3; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the sticky error word of the current device (nullptr and
// a recorded error if the runtime call fails).
unsigned int* device_error_word();

// The process-wide pa_decode_select mode (its prefill bits included).
int decode_select_mode();

// Per-device cache of a __device__ symbol's address.  An entry is keyed on
// the device's current context as well, so it is looked up again after a
// cudaDeviceReset (the next context may load the module elsewhere).
struct SymbolCache {
    std::mutex mu;
    const void* ctx[256] = {};
    void* addr[256] = {};
};

// Address of `symbol` on the current device (nullptr and a recorded error if
// a runtime call fails).
void* symbol_address(const void* symbol, SymbolCache* cache, const char* what);

// Translate a CUDA runtime error into PA_ERR_CUDA with context.
pa_status cuda_fail(int err, const char* what);

// pa_decode with the shared-prefix switches (decode_host.cu): partitions
// below prefix_parts of sequences whose table starts with row 0's blocks are
// left to the caller's prefix records; force_ws sends every record through
// the workspace and always runs the merge.  With fuse_prefix_blocks > 0 one
// CTA per (sequence, kv head) reads the suffix past that many blocks and
// merges the prefix_parts records itself (no merge kernel).
pa_status decode_impl(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                      const void* value_cache, pa_dtype cache_dt, const int32_t* block_tables,
                      int MB, const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs,
                      int64_t NB, int max_ctx, float scale, float k_scale, float v_scale,
                      int partition, void* workspace, size_t workspace_bytes, pa_stream_t stream,
                      int prefix_parts, int force_ws, int fuse_prefix_blocks);

// Shared-prefix decode, step 1 (prefill.cu): split-K records (m, l, o * v_scale)
// of partitions 0 .. prefix_tokens / chunk_tokens - 1 of every (sequence, head),
// from K/V in 16-bit `dt` at k_src / v_src (blocks named by table_row0, or
// blocks 0.. when it is NULL).  sl = scale * k_scale * log2(e).
pa_status prefix_records(const void* q, pa_dtype dt, const void* k_src, const void* v_src,
                         int64_t src_blocks, const int32_t* table_row0, int S, int Hq, int Hkv,
                         int D, int bs, int prefix_tokens, int chunk_tokens, float sl,
                         float v_scale, float2* ws_ml, float* ws_o, int max_parts,
                         pa_stream_t stream);

}  // namespace pa
