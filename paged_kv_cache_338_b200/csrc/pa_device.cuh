// Device helpers: storage conversions, the 128-byte TMA swizzle, and thin
// inline-PTX wrappers for mbarriers and tensor-map (TMA) bulk loads on sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <utility>

#include "pa.h"

namespace pa {

// Count one kernel enqueued by this library (pa_launch_count()).
void note_launch();

namespace dev {

// ------------------------------------------------------------ storage types
template <int DT> struct Storage;
template <> struct Storage<PA_F32> { using T = float; static constexpr int bytes = 4; };
template <> struct Storage<PA_F16> { using T = __half; static constexpr int bytes = 2; };
template <> struct Storage<PA_BF16> { using T = __nv_bfloat16; static constexpr int bytes = 2; };
template <> struct Storage<PA_FP8_E4M3> { using T = uint8_t; static constexpr int bytes = 1; };

// Expand one 16-byte chunk of storage into 16 / bytes floats (exact widening).
template <int DT> struct Chunk;

template <> struct Chunk<PA_F32> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void to_float(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
    }
};

template <> struct Chunk<PA_BF16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void pair(uint32_t u, float* f) {
        f[0] = __uint_as_float(u << 16);          // low half is the lower-indexed element
        f[1] = __uint_as_float(u & 0xffff0000u);
    }
    __device__ __forceinline__ static void to_float(const uint4& r, float* f) {
        pair(r.x, f); pair(r.y, f + 2); pair(r.z, f + 4); pair(r.w, f + 6);
    }
};

template <> struct Chunk<PA_F16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void pair(uint32_t u, float* f) {
        __half2 h = *reinterpret_cast<__half2*>(&u);
        float2 v = __half22float2(h);
        f[0] = v.x; f[1] = v.y;
    }
    __device__ __forceinline__ static void to_float(const uint4& r, float* f) {
        pair(r.x, f); pair(r.y, f + 2); pair(r.z, f + 4); pair(r.w, f + 6);
    }
};

template <> struct Chunk<PA_FP8_E4M3> {
    static constexpr int N = 16;
    // two E4M3 codes -> two halves (exact: every E4M3 value is a normal f16)
    __device__ __forceinline__ static void pair(uint16_t u, float* f) {
        __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(u), __NV_E4M3);
        float2 v = __half22float2(*reinterpret_cast<__half2*>(&h));
        f[0] = v.x; f[1] = v.y;
    }
    __device__ __forceinline__ static void word(uint32_t u, float* f) {
        pair(static_cast<uint16_t>(u & 0xffffu), f);
        pair(static_cast<uint16_t>(u >> 16), f + 2);
    }
    __device__ __forceinline__ static void to_float(const uint4& r, float* f) {
        word(r.x, f); word(r.y, f + 4); word(r.z, f + 8); word(r.w, f + 12);
    }
};

// Load one element of a q / out dtype as float, and round a float into it.
template <int QT> __device__ __forceinline__ float load_q(const void* p, size_t i);
template <> __device__ __forceinline__ float load_q<PA_F32>(const void* p, size_t i) {
    return static_cast<const float*>(p)[i];
}
template <> __device__ __forceinline__ float load_q<PA_F16>(const void* p, size_t i) {
    return __half2float(static_cast<const __half*>(p)[i]);
}
template <> __device__ __forceinline__ float load_q<PA_BF16>(const void* p, size_t i) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

template <int QT> __device__ __forceinline__ void store_out(void* p, size_t i, float v);
template <> __device__ __forceinline__ void store_out<PA_F32>(void* p, size_t i, float v) {
    static_cast<float*>(p)[i] = v;
}
template <> __device__ __forceinline__ void store_out<PA_F16>(void* p, size_t i, float v) {
    static_cast<__half*>(p)[i] = __float2half_rn(v);
}
template <> __device__ __forceinline__ void store_out<PA_BF16>(void* p, size_t i, float v) {
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

// -------------------------------------------------------------- swizzle
// Byte offset of 16-byte chunk c of 128-byte row r inside a tile written by a
// tensor-map load with CU_TENSOR_MAP_SWIZZLE_128B (tile base 1024-aligned):
// the chunk index is XORed with the row index modulo 8.
__device__ __forceinline__ uint32_t swz128(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete, for at most
// `limit_ns` nanoseconds.  Returns false on timeout (the caller records it).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns = 2000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        #pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// 4-D tiled tensor-map load into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
        : "memory");
}

// Untiled bulk copy global -> shared memory, completing on `bar` (both
// addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start
// launching (it still waits for this grid's memory with grid_dependency_wait).
__device__ __forceinline__ void launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch `kern` as a programmatic dependent of the kernel before it in the
// stream: its CTAs may become resident while that kernel finishes, and must
// call grid_dependency_wait() before touching memory the stream wrote.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e == cudaSuccess) note_launch();
    return e;
}

// Opt kernel Kern in to `bytes` of dynamic shared memory on the current device.
// The attribute belongs to the kernel in each device's context; a driver call
// per launch costs microseconds of host time, so the largest size already set
// is remembered per device and a launch that needs no more skips the call.
template <auto Kern>
inline cudaError_t ensure_dynamic_smem(size_t bytes) {
    constexpr int kDevices = 64;
    static std::atomic<int> set_bytes[kDevices] = {};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices)
        return cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (set_bytes[dev].load(std::memory_order_acquire) >= (int)bytes) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) {
        int cur = set_bytes[dev].load(std::memory_order_relaxed);
        while (cur < (int)bytes &&
               !set_bytes[dev].compare_exchange_weak(cur, (int)bytes, std::memory_order_release))
        {
        }
    }
    return e;
}

// cudaOccupancyMaxActiveBlocksPerMultiprocessor for kernel Kern, remembered
// per device for the last shared-memory size asked (the launchers ask the same
// sizes call after call).
template <auto Kern>
inline cudaError_t occupancy(int* per_sm, int threads, size_t smem) {
    constexpr int kDevices = 64;
    static std::atomic<unsigned long long> memo[kDevices] = {};   // (smem + 1) << 32 | blocks
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices)
        return cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, Kern, threads, smem);
    const unsigned long long m = memo[dev].load(std::memory_order_acquire);
    if ((m >> 32) == (unsigned long long)smem + 1) {
        *per_sm = (int)(m & 0xffffffffu);
        return cudaSuccess;
    }
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, Kern, threads, smem);
    if (e == cudaSuccess)
        memo[dev].store((((unsigned long long)smem + 1) << 32) | (unsigned)*per_sm,
                        std::memory_order_release);
    return e;
}

// 5-D tiled tensor-map load into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar),
          "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Bring one 128-byte line of global memory into L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(ptr)) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Sticky device error bits (see pa.h).
__device__ __forceinline__ void raise_error(unsigned int* word, unsigned int bit) {
    if (word) atomicOr(word, bit);
}

}  // namespace dev
}  // namespace pa
