// Library-wide plumbing (error reporting, the device error word) and the two
// memory-movement steps of a decode step: the cache append and the
// copy-on-write block copy.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_set>
#include <vector>

#include "pa_device.cuh"
#include "pa_internal.h"

// One sticky error word per device; kernels get its address as a parameter.
static __device__ unsigned int g_pa_device_error;

namespace pa {

static thread_local std::string t_error;

pa_status fail(pa_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_error = buf;
    return st;
}

void clear_error() { t_error.clear(); }

static std::atomic<unsigned long long> g_launches{0};

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

pa_status cuda_fail(int err, const char* what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(static_cast<cudaError_t>(err)));
}

// The calling thread's current CUDA context (nullptr before the runtime has
// made one current), through the driver entry point the runtime exposes.
static const void* current_context() {
    using Fn = CUresult (*)(CUcontext*);
    static Fn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<Fn>(p);
    });
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

void* symbol_address(const void* symbol, SymbolCache* cache, const char* what) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { cuda_fail(e, "cudaGetDevice"); return nullptr; }
    if (dev < 0 || dev >= 256) { fail(PA_ERR_CUDA, "device ordinal %d", dev); return nullptr; }
    std::lock_guard<std::mutex> lk(cache->mu);
    const void* ctx = current_context();
    if (!cache->addr[dev] || !ctx || cache->ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, symbol);    // makes the device's context current
        if (e != cudaSuccess) { cuda_fail(e, what); return nullptr; }
        cache->addr[dev] = p;
        cache->ctx[dev] = current_context();
    }
    return cache->addr[dev];
}

unsigned int* device_error_word() {
    static SymbolCache cache;
    return static_cast<unsigned int*>(
        symbol_address(&g_pa_device_error, &cache, "cudaGetSymbolAddress(error word)"));
}

namespace {

// ------------------------------------------------------------ cache append
// One thread per 16-byte chunk of a (token, kv head) row of the input.
// Same dtype: the chunk is copied.  fp8 cache: 8 input elements become 8
// E4M3 codes (x / scale in binary32, round to nearest even, saturate).
template <int IN, bool TO_FP8>
__global__ void reshape_and_cache_kernel(const uint8_t* __restrict__ key,
                                         const uint8_t* __restrict__ value,
                                         uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                                         const int64_t* __restrict__ slots, int T, int HkvD,
                                         int64_t nslots, float k_scale, float v_scale,
                                         unsigned int* err) {
    dev::grid_dependency_wait();       // launched as a dependent of the kernel before it
    dev::launch_dependents();
    constexpr int ein = dev::Storage<IN>::bytes;
    constexpr int per = TO_FP8 ? 8 : 16 / ein;                 // elements per thread
    const int per_row = HkvD / per;
    const int64_t total = (int64_t)T * per_row;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / per_row);
        const int c = (int)(i % per_row);
        const int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= nslots) {
            dev::raise_error(err, PA_DEV_BAD_SLOT);
            continue;
        }
        const size_t src = ((size_t)t * HkvD + (size_t)c * per) * ein;
        if constexpr (!TO_FP8) {
            const size_t dst = ((size_t)slot * HkvD + (size_t)c * per) * ein;
            *reinterpret_cast<uint4*>(kc + dst) = *reinterpret_cast<const uint4*>(key + src);
            *reinterpret_cast<uint4*>(vc + dst) = *reinterpret_cast<const uint4*>(value + src);
        } else {
            const size_t dst = (size_t)slot * HkvD + (size_t)c * per;
            #pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint8_t* in = which ? value : key;
                const float sc = which ? v_scale : k_scale;
                float x[8];
                if constexpr (IN == PA_F32) {
                    const uint4 a = *reinterpret_cast<const uint4*>(in + src);
                    const uint4 b = *reinterpret_cast<const uint4*>(in + src + 16);
                    dev::Chunk<PA_F32>::to_float(a, x);
                    dev::Chunk<PA_F32>::to_float(b, x + 4);
                } else {
                    dev::Chunk<IN>::to_float(*reinterpret_cast<const uint4*>(in + src), x);
                }
                uint32_t w[2];
                #pragma unroll
                for (int k = 0; k < 2; ++k) {
                    uint32_t acc = 0;
                    #pragma unroll
                    for (int j = 0; j < 4; j += 2) {
                        float2 y = make_float2(__fdiv_rn(x[4 * k + j], sc),
                                               __fdiv_rn(x[4 * k + j + 1], sc));
                        __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
                        acc |= (uint32_t)c2 << (16 * (j / 2));
                    }
                    w[k] = acc;
                }
                *reinterpret_cast<uint2*>((which ? vc : kc) + dst) = make_uint2(w[0], w[1]);
            }
        }
    }
}

template <int IN, bool TO_FP8>
cudaError_t launch_append(const void* key, const void* value, void* kc, void* vc,
                          const int64_t* slots, int T, int HkvD, int64_t nslots, float ks,
                          float vs, unsigned int* err, cudaStream_t st) {
    constexpr int per = TO_FP8 ? 8 : 16 / dev::Storage<IN>::bytes;
    const int64_t total = (int64_t)T * (HkvD / per);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return dev::launch_pdl(reshape_and_cache_kernel<IN, TO_FP8>, dim3((unsigned)blocks),
                           dim3(threads), 0, st, static_cast<const uint8_t*>(key),
                           static_cast<const uint8_t*>(value), static_cast<uint8_t*>(kc),
                           static_cast<uint8_t*>(vc), slots, T, HkvD, nslots, ks, vs, err);
}

// ------------------------------------------------------------- block copy
constexpr int kMaxPairsPerLaunch = 1024;   // 8 KB of kernel parameters

struct CopyList {
    int n;
    int2 pair[kMaxPairsPerLaunch];
};

// blockIdx.x = pair, blockIdx.y = 0 (K) / 1 (V); 16-byte vectors.  The host
// has checked that no destination is also a source, so each thread loads a
// batch of vectors before it stores any (a plain load-store loop would keep
// one load in flight per thread).
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint8_t* __restrict__ kc,
                                                          uint8_t* __restrict__ vc, size_t block_bytes,
                                                          const __grid_constant__ CopyList list) {
    constexpr int kBatch = 8;
    dev::grid_dependency_wait();       // launched as a dependent of the kernel before it
    dev::launch_dependents();
    const int2 pr = list.pair[blockIdx.x];
    uint8_t* base = blockIdx.y ? vc : kc;
    const uint4* src = reinterpret_cast<const uint4*>(base + (size_t)pr.x * block_bytes);
    uint4* dst = reinterpret_cast<uint4*>(base + (size_t)pr.y * block_bytes);
    const size_t n16 = block_bytes / 16;
    for (size_t i0 = threadIdx.x; i0 < n16; i0 += (size_t)kBatch * blockDim.x) {
        uint4 r[kBatch];
        #pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const size_t i = i0 + (size_t)u * blockDim.x;
            if (i < n16) r[u] = src[i];
        }
        #pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const size_t i = i0 + (size_t)u * blockDim.x;
            if (i < n16) dst[i] = r[u];
        }
    }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" const char* pa_last_error(void) { return t_error.c_str(); }

extern "C" int pa_version(void) { return 10000; }

extern "C" uint64_t pa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" pa_status pa_device_status(unsigned int* bits, int clear, pa_stream_t stream) {
    PA_NVTX_RANGE("pa_device_status");
    clear_error();
    if (!bits) return fail(PA_ERR_INVALID_ARG, "bits is NULL");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0;
    e = cudaMemcpyFromSymbolAsync(&v, g_pa_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (clear && v) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbolAsync(g_pa_device_error, &zero, sizeof(zero), 0,
                                    cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    }
    *bits = v;
    return PA_OK;
}

extern "C" pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype in_dt,
                                          void* key_cache, void* value_cache, pa_dtype cache_dt,
                                          const int64_t* slot_mapping, int T, int Hkv, int D,
                                          int bs, int64_t NB, float k_scale, float v_scale,
                                          pa_stream_t stream) {
    PA_NVTX_RANGE("pa_reshape_and_cache");
    clear_error();
    if (!valid_dtype(in_dt) || !valid_dtype(cache_dt)) return fail(PA_ERR_INVALID_ARG, "bad dtype");
    if (T < 0 || Hkv <= 0 || D <= 0 || bs <= 0 || NB <= 0)
        return fail(PA_ERR_INVALID_ARG, "negative or zero size");
    if (!(std::isfinite(k_scale) && k_scale > 0 && std::isfinite(v_scale) && v_scale > 0))
        return fail(PA_ERR_INVALID_ARG, "scales must be finite and > 0");
    const bool to_fp8 = cache_dt == PA_FP8_E4M3 && in_dt != PA_FP8_E4M3;
    if (!(in_dt == cache_dt || to_fp8))
        return fail(PA_ERR_UNSUPPORTED, "append from dtype %d into dtype %d", in_dt, cache_dt);
    if (cache_dt != PA_FP8_E4M3 && (k_scale != 1.f || v_scale != 1.f))
        return fail(PA_ERR_INVALID_ARG, "k_scale / v_scale apply to fp8 caches only");
    const int ein = elem_size(in_dt);
    if (((int64_t)D * ein) % 16 || (to_fp8 && D % 8))
        return fail(PA_ERR_UNSUPPORTED, "D * element size must be a multiple of 16 bytes");
    if (T == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    unsigned int* err = device_error_word();
    if (!err) return PA_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int HkvD = Hkv * D;
    const int64_t nslots = NB * bs;
    cudaError_t e;
    if (!to_fp8) {
        switch (ein) {
        case 4: e = launch_append<PA_F32, false>(key, value, key_cache, value_cache, slot_mapping,
                                                  T, HkvD, nslots, 1.f, 1.f, err, st); break;
        case 2: e = launch_append<PA_F16, false>(key, value, key_cache, value_cache, slot_mapping,
                                                  T, HkvD, nslots, 1.f, 1.f, err, st); break;
        default: e = launch_append<PA_FP8_E4M3, false>(key, value, key_cache, value_cache,
                                                        slot_mapping, T, HkvD, nslots, 1.f, 1.f,
                                                        err, st); break;
        }
    } else {
        switch (in_dt) {
        case PA_F32: e = launch_append<PA_F32, true>(key, value, key_cache, value_cache,
                                                     slot_mapping, T, HkvD, nslots, k_scale,
                                                     v_scale, err, st); break;
        case PA_F16: e = launch_append<PA_F16, true>(key, value, key_cache, value_cache,
                                                     slot_mapping, T, HkvD, nslots, k_scale,
                                                     v_scale, err, st); break;
        default: e = launch_append<PA_BF16, true>(key, value, key_cache, value_cache,
                                                  slot_mapping, T, HkvD, nslots, k_scale,
                                                  v_scale, err, st); break;
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
    return PA_OK;
}

extern "C" pa_status pa_copy_blocks(void* key_cache, void* value_cache, size_t block_bytes,
                                    int64_t NB, const int32_t* pairs, int n, pa_stream_t stream) {
    PA_NVTX_RANGE("pa_copy_blocks");
    clear_error();
    if (n < 0 || NB <= 0 || block_bytes == 0 || block_bytes % 16)
        return fail(PA_ERR_INVALID_ARG, "bad sizes (block_bytes must be a positive multiple of 16)");
    if (n == 0) return PA_OK;
    if (!key_cache || !value_cache || !pairs) return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(key_cache) || !aligned16(value_cache))
        return fail(PA_ERR_INVALID_ARG, "caches must be 16-byte aligned");
    std::unordered_set<int32_t> dsts, srcs;
    dsts.reserve(2 * (size_t)n);
    srcs.reserve(2 * (size_t)n);
    for (int i = 0; i < n; ++i) {
        const int32_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= NB || d < 0 || d >= NB)
            return fail(PA_ERR_INVALID_ARG, "pair %d (%d -> %d) outside [0, %lld)", i, s, d,
                        (long long)NB);
        if (!dsts.insert(d).second) return fail(PA_ERR_INVALID_ARG, "destination %d repeats", d);
        srcs.insert(s);
    }
    for (int32_t d : dsts)
        if (srcs.count(d)) return fail(PA_ERR_INVALID_ARG, "block %d is both source and destination", d);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    for (int off = 0; off < n; off += kMaxPairsPerLaunch) {
        CopyList list;
        list.n = n - off < kMaxPairsPerLaunch ? n - off : kMaxPairsPerLaunch;
        for (int i = 0; i < list.n; ++i)
            list.pair[i] = make_int2(pairs[2 * (off + i)], pairs[2 * (off + i) + 1]);
        cudaError_t e = dev::launch_pdl(copy_blocks_kernel, dim3((unsigned)list.n, 2), dim3(256), 0,
                                        st, static_cast<uint8_t*>(key_cache),
                                        static_cast<uint8_t*>(value_cache), block_bytes, list);
        if (e != cudaSuccess) return cuda_fail(e, "copy_blocks launch");
    }
    return PA_OK;
}
