// Shared-prefix ("cascade") decode: many sequences whose block tables start
// with the same physical blocks -- a common system prompt, or the prefix the
// block pool shares by reference ("01. PagedAttention 详解" §6 and summary:
// requests share blocks of a common prefix; "PagedAttention 机制" §5.3.2) --
// attend to that prefix with one tensor-core pass over all their queries,
// instead of each sequence reading and converting the same K/V again.
//
// Attention splits over key ranges exactly (the split-K identity the decode
// merge already uses), so the step is:
//   1. (fp8 cache) the prefix blocks, converted exactly to the q dtype: every
//      E4M3 value is a 16-bit float; the scales stay separate;
//   2. the prefix kernel: for every (sequence, query head), the record
//      (m, l, o) of each prefix chunk, with all sequences' queries as the
//      rows of 128-row tensor-core tiles (prefill kernel, prefix mode);
//   3. the decode kernel over the private suffixes.  Suffixes of up to 4096
//      tokens: one CTA per (sequence, kv head) reads the whole suffix and
//      merges the prefix records in its epilogue.  Longer: partitions of the
//      chunk size past the prefix, then
//   4. the split-K merge of all records.
//   Either way a sequence whose table does not start with row 0's prefix
//   blocks, or that is shorter than the prefix, reads its own prefix blocks
//   (and, split, blanks the prefix kernel's records for it).
// The result is pa_decode's, up to rounding order.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace {

constexpr int kChunkTokens = 256;     // prefix tokens per record (a decode partition)

// Prefix blocks of table row 0 -> 16-bit copies (exact: E4M3 -> f16 -> QT).
// grid (chunks of the block, prefix blocks, 2 for K and V); 8 codes a thread.
template <int QT>
__global__ void prefix_to_16bit(const uint8_t* kc, const uint8_t* vc, const int32_t* table_row0,
                                int64_t NB, int blk_elems, uint16_t* sk, uint16_t* sv,
                                unsigned int* err) {
    // a programmatic dependent of the cache append: wait for its memory, and
    // let the prefix kernel's CTAs get resident meanwhile
    pa::dev::grid_dependency_wait();
    pa::dev::launch_dependents();
    const int lb = blockIdx.y;
    const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (e >= blk_elems) return;
    const int32_t id = table_row0[lb];
    const uint8_t* src = blockIdx.z ? vc : kc;
    uint16_t* dst = (blockIdx.z ? sv : sk) + (size_t)lb * blk_elems + e;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (id >= 0 && id < NB) {
        const uint2 codes = *reinterpret_cast<const uint2*>(src + (size_t)id * blk_elems + e);
        uint32_t w[4];
        const uint32_t c[2] = {codes.x, codes.y};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint16_t pair = static_cast<uint16_t>(c[i >> 1] >> (16 * (i & 1)));
            __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair),
                                                       __NV_E4M3);
            if constexpr (QT == PA_F16) {
                w[i] = static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
            } else {
                const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h));
                __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);   // exact
                w[i] = *reinterpret_cast<uint32_t*>(&b);
            }
        }
        out = make_uint4(w[0], w[1], w[2], w[3]);
    } else if (e == 0 && blockIdx.z == 0) {
        atomicOr(err, PA_DEV_BAD_BLOCK);
    }
    *reinterpret_cast<uint4*>(dst) = out;
}

int chunk_for(int prefix_tokens) {
    if (prefix_tokens % kChunkTokens == 0) return kChunkTokens;
    if (prefix_tokens % 128 == 0) return 128;
    return prefix_tokens;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Suffixes of at most this many tokens are read by one CTA per (sequence, kv
// head), which also merges the prefix records (no merge kernel); longer ones
// are split into chunk-sized partitions and merged by the split-K merge.
constexpr int kFusedSuffixMax = 4096;

bool fused(int max_ctx, int prefix_tokens) { return max_ctx - prefix_tokens <= kFusedSuffixMax; }

// Records per (sequence, head): fused, the prefix chunks; split, those max_ctx
// needs and at least one past the prefix (an irregular sequence's first
// suffix CTA writes it).
int64_t parts(int max_ctx, int chunk, int prefix_tokens) {
    const int64_t k = prefix_tokens / chunk;
    if (fused(max_ctx, prefix_tokens)) return k;
    const int64_t need = max_ctx <= chunk ? 1 : ((int64_t)max_ctx + chunk - 1) / chunk;
    return need > k + 1 ? need : k + 1;
}

}  // namespace

using pa::fail;

extern "C" pa_status pa_decode_shared_prefix_workspace_size(int S, int Hq, int Hkv, int D, int bs,
                                                            int max_ctx, int prefix_tokens,
                                                            pa_dtype cache_dt, size_t* bytes) {
    pa::clear_error();
    if (!bytes) return fail(PA_ERR_INVALID_ARG, "bytes is NULL");
    if (S < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || max_ctx < 0 || prefix_tokens <= 0 ||
        prefix_tokens % bs)
        return fail(PA_ERR_INVALID_ARG, "bad sizes (prefix_tokens a positive multiple of bs)");
    *bytes = 0;
    if (S == 0 || max_ctx < prefix_tokens) return PA_OK;     // plain decode, no workspace
    const int chunk = chunk_for(prefix_tokens);
    const int64_t mp = parts(max_ctx, chunk, prefix_tokens);
    size_t b = align256((size_t)S * Hq * mp * (sizeof(float) * 2 + sizeof(float) * D));
    if (cache_dt == PA_FP8_E4M3)
        b += 2 * align256((size_t)prefix_tokens * Hkv * D * 2);
    *bytes = b;
    return PA_OK;
}

extern "C" pa_status pa_decode_shared_prefix(void* out, const void* q, pa_dtype q_dt,
                                             const void* key_cache, const void* value_cache,
                                             pa_dtype cache_dt, const int32_t* block_tables,
                                             int MB, const int32_t* context_lens, int S, int Hq,
                                             int Hkv, int D, int bs, int64_t NB, int max_ctx,
                                             float scale, float k_scale, float v_scale,
                                             int prefix_tokens, void* workspace,
                                             size_t workspace_bytes, pa_stream_t stream) {
    PA_NVTX_RANGE("pa_decode_shared_prefix");
    pa::clear_error();
    if (!pa::valid_dtype(q_dt) || !pa::valid_dtype(cache_dt))
        return fail(PA_ERR_INVALID_ARG, "bad dtype");
    if (q_dt != PA_F16 && q_dt != PA_BF16)
        return fail(PA_ERR_UNSUPPORTED, "shared-prefix decode takes f16 or bf16 queries");
    if (cache_dt != q_dt && cache_dt != PA_FP8_E4M3)
        return fail(PA_ERR_UNSUPPORTED, "cache dtype %d with q dtype %d", cache_dt, q_dt);
    if (D != 64 && D != 128) return fail(PA_ERR_UNSUPPORTED, "head size %d (64 or 128)", D);
    if (D * pa::elem_size(cache_dt) < 128)      // the decode kernel's 128-byte row segments
        return fail(PA_ERR_UNSUPPORTED, "head size %d with this cache dtype", D);
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(PA_ERR_INVALID_ARG, "bad head counts");
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(PA_ERR_UNSUPPORTED, "group size %d (1, 2, 4, 8 or 16)", G);
    if (bs != 8 && bs != 16 && bs != 32) return fail(PA_ERR_UNSUPPORTED, "block size %d", bs);
    if (prefix_tokens <= 0 || prefix_tokens % bs || (int64_t)prefix_tokens > (int64_t)MB * bs)
        return fail(PA_ERR_INVALID_ARG, "prefix_tokens %d: a positive multiple of bs within MB * bs",
                    prefix_tokens);
    if (!(std::isfinite(scale) && scale > 0.f))
        return fail(PA_ERR_INVALID_ARG, "scale must be finite and positive");
    if (S < 0 || max_ctx < 0 || NB <= 0 || NB > 0x7fffffffLL)
        return fail(PA_ERR_INVALID_ARG, "bad sizes");
    if (S == 0) return PA_OK;
    if (max_ctx < prefix_tokens)        // no sequence can hold the prefix: a plain decode
        return pa::decode_impl(out, q, q_dt, key_cache, value_cache, cache_dt, block_tables, MB,
                               context_lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale, k_scale,
                               v_scale, 0, nullptr, 0, stream, 0, 0, 0);
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    size_t need = 0;
    pa_status st = pa_decode_shared_prefix_workspace_size(S, Hq, Hkv, D, bs, max_ctx,
                                                          prefix_tokens, cache_dt, &need);
    if (st) return st;
    if (!workspace || workspace_bytes < need || !pa::aligned16(workspace))
        return fail(PA_ERR_INVALID_ARG, "workspace needs %zu bytes, 16-byte aligned (got %zu)",
                    need, workspace_bytes);
    const int chunk = chunk_for(prefix_tokens);
    const int64_t mp = parts(max_ctx, chunk, prefix_tokens);
    if (mp > 65535) return fail(PA_ERR_UNSUPPORTED, "too many partitions");
    char* w = static_cast<char*>(workspace);
    float2* ws_ml = reinterpret_cast<float2*>(w);
    float* ws_o = reinterpret_cast<float*>(w + sizeof(float2) * (size_t)S * Hq * mp);
    const size_t rec_bytes = align256((size_t)S * Hq * mp * (sizeof(float) * 2 + sizeof(float) * D));

    const void* k_src = key_cache;
    const void* v_src = value_cache;
    int64_t src_blocks = NB;
    const int32_t* table = block_tables;                 // row 0
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (cache_dt == PA_FP8_E4M3) {
        const int nblk = prefix_tokens / bs;
        const int blk_elems = bs * Hkv * D;
        const size_t half = align256((size_t)prefix_tokens * Hkv * D * 2);
        uint16_t* sk = reinterpret_cast<uint16_t*>(w + rec_bytes);
        uint16_t* sv = reinterpret_cast<uint16_t*>(w + rec_bytes + half);
        unsigned int* err = pa::device_error_word();
        if (!err) return PA_ERR_CUDA;
        const dim3 grid((unsigned)((blk_elems / 8 + 255) / 256), (unsigned)nblk, 2);
        const uint8_t* kc8 = static_cast<const uint8_t*>(key_cache);
        const uint8_t* vc8 = static_cast<const uint8_t*>(value_cache);
        cudaError_t e = q_dt == PA_BF16
                            ? pa::dev::launch_pdl(prefix_to_16bit<PA_BF16>, grid, dim3(256), 0, cs,
                                                  kc8, vc8, block_tables, NB, blk_elems, sk, sv, err)
                            : pa::dev::launch_pdl(prefix_to_16bit<PA_F16>, grid, dim3(256), 0, cs,
                                                  kc8, vc8, block_tables, NB, blk_elems, sk, sv, err);
        if (e != cudaSuccess) return pa::cuda_fail(e, "prefix conversion launch");
        k_src = sk;
        v_src = sv;
        src_blocks = nblk;
        table = nullptr;                                 // blocks 0.. of the copy
    }
    const float sl = (float)((double)scale * (double)k_scale * 1.4426950408889634);
    st = pa::prefix_records(q, q_dt, k_src, v_src, src_blocks, table, S, Hq, Hkv, D, bs,
                            prefix_tokens, chunk, sl, cache_dt == PA_FP8_E4M3 ? v_scale : 1.f,
                            ws_ml, ws_o, (int)mp, stream);
    if (st) return st;
    if (fused(max_ctx, prefix_tokens))
        return pa::decode_impl(out, q, q_dt, key_cache, value_cache, cache_dt, block_tables, MB,
                               context_lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale, k_scale,
                               v_scale, chunk, workspace, rec_bytes, stream, prefix_tokens / chunk,
                               0, prefix_tokens / bs);
    return pa::decode_impl(out, q, q_dt, key_cache, value_cache, cache_dt, block_tables, MB,
                           context_lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale, k_scale, v_scale,
                           chunk, workspace, rec_bytes, stream, prefix_tokens / chunk, 1, 0);
}
