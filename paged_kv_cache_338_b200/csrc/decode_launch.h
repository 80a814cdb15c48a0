// Launch descriptors shared by the host code of pa_decode and the per-dtype
// instantiation units of the decode kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "decode_kernels.cuh"

namespace pa {
namespace dec {

struct Launch {
    CUtensorMap tmk, tmv;
    Params p;
    int bs, D;
    bool pair;     // two 8-token blocks per 16-token stage
    int hg;        // kv heads per CTA (1, or 4 with the tensor-core consumer)
    int gc;        // SIMT: query heads per CTA
    bool mma;      // tensor-core consumer
    int mrows;     // MMA: 8 or 16 query rows
    dim3 grid;
    cudaStream_t stream;
    bool balanced; // persistent work-balanced kernel (grid computed at launch)
    int G;         // query heads per kv head
    int num_sms;
};

constexpr int kMaxBalancedCtas = 1024;   // the workspace layout assumes at most this many

// cudaErrorNotSupported when no kernel is built for the combination.
cudaError_t launch_f32(const Launch& L);
cudaError_t launch_f16(const Launch& L);
cudaError_t launch_bf16(const Launch& L);
cudaError_t launch_fp8_q_f16(const Launch& L);
cudaError_t launch_fp8_q_bf16(const Launch& L);

template <class C>
cudaError_t launch_one(const Launch& L) {
    if constexpr (C::PER != 1 || C::HG != 1) {
        // the host pairs blocks and groups heads for the partition kernel only
        if (L.balanced) return cudaErrorNotSupported;
    } else if (L.balanced) {
        auto kern = decode_balanced<C>;
        const int smem = static_cast<int>(BalancedSmem<C>::bytes(L.mma ? L.G : L.gc));
        cudaError_t e = dev::ensure_dynamic_smem<decode_balanced<C>>((size_t)smem);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        e = dev::occupancy<decode_balanced<C>>(&per_sm, C::THREADS, (size_t)smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        int ctas = per_sm * L.num_sms;
        if (ctas > kMaxBalancedCtas) ctas = kMaxBalancedCtas;
        if (L.p.whole_items) {
            // whole items: groups of one CTA per (kv head, head chunk)
            const int hc = L.p.Hkv * (C::MMA ? 1 : L.G / C::GC);
            ctas = ctas >= hc ? ctas / hc * hc : hc;
        }
        return dev::launch_pdl(kern, dim3((unsigned)ctas), dim3(C::THREADS), (size_t)smem,
                               L.stream, L.tmk, L.tmv, L.p);
    }
    Params p = L.p;
    if constexpr (C::MMA) if (p.part_group > 1) {
        // Grouped partitions need a warp-merge area of their own; use them
        // only if it costs no resident CTA per SM.
        auto kern = decode_partition<C, true>;
        const size_t big = C::SMEM + group_merge_bytes<C>(L.G);
        cudaError_t e = dev::ensure_dynamic_smem<decode_partition<C, true>>(big);
        if (e != cudaSuccess) return e;
        int occ1 = 0, occ2 = 0;
        e = dev::occupancy<decode_partition<C, false>>(&occ1, C::THREADS, C::SMEM);
        if (e != cudaSuccess) return e;
        e = dev::occupancy<decode_partition<C, true>>(&occ2, C::THREADS, big);
        if (e != cudaSuccess) return e;
        if (occ2 >= occ1 && occ2 > 0) {
            return dev::launch_pdl(kern, L.grid, dim3(C::THREADS), big, L.stream, L.tmk, L.tmv,
                                   p);
        }
    }
    // one partition per CTA
    dim3 grid = L.grid;
    if (p.part_group > 1) {
        p.part_group = 1;
        (p.heads_fastest ? grid.y : grid.x) = (unsigned)p.max_parts;
    }
    auto kern = decode_partition<C, false>;
    const size_t smem = C::SMEM + (size_t)p.rec_smem;   // + the shared-prefix records
    // opt in to > 48 KB of dynamic shared memory
    cudaError_t e = dev::ensure_dynamic_smem<decode_partition<C, false>>(smem);
    if (e != cudaSuccess) return e;
    return dev::launch_pdl(kern, grid, dim3(C::THREADS), smem, L.stream, L.tmk, L.tmv, p);
}

template <int DT, int D>
constexpr bool row_ok() {
    return D * dev::Storage<DT>::bytes == 128 || D * dev::Storage<DT>::bytes == 256 ||
           D * dev::Storage<DT>::bytes == 512;
}

// BS: tokens per stage; PB: tokens per physical block (BS / PB blocks a stage)
template <int DT, int QT, int BS, int D, int PB>
cudaError_t launch_by_heads(const Launch& L) {
    if constexpr (!row_ok<DT, D>()) {
        return cudaErrorNotSupported;
    } else {
        if (L.mma) {
            if constexpr (((DT == QT && (DT == PA_F16 || DT == PA_BF16)) || DT == PA_FP8_E4M3) &&
                          D <= 128) {
                if (L.hg == 4) {
                    if (L.mrows == 8) return launch_one<Cfg<DT, QT, BS, D, 8, true, 8, PB, 4>>(L);
                    return launch_one<Cfg<DT, QT, BS, D, 16, true, 16, PB, 4>>(L);
                }
                if (L.mrows == 8) return launch_one<Cfg<DT, QT, BS, D, 8, true, 8, PB>>(L);
                return launch_one<Cfg<DT, QT, BS, D, 16, true, 16, PB>>(L);
            } else {
                return cudaErrorNotSupported;
            }
        }
        switch (L.gc) {
        case 1: return launch_one<Cfg<DT, QT, BS, D, 1, false, 8, PB>>(L);
        case 2: return launch_one<Cfg<DT, QT, BS, D, 2, false, 8, PB>>(L);
        case 4:
            if constexpr (D <= 128) return launch_one<Cfg<DT, QT, BS, D, 4, false, 8, PB>>(L);
            else return cudaErrorNotSupported;
        }
        return cudaErrorNotSupported;
    }
}

template <int DT, int QT, int BS, int PB>
cudaError_t launch_by_dim(const Launch& L) {
    switch (L.D) {
    case 64: return launch_by_heads<DT, QT, BS, 64, PB>(L);
    case 128: return launch_by_heads<DT, QT, BS, 128, PB>(L);
    case 256: return launch_by_heads<DT, QT, BS, 256, PB>(L);
    }
    return cudaErrorNotSupported;
}

template <int DT, int QT>
cudaError_t launch_dtype(const Launch& L) {
    switch (L.bs) {
    case 8: return L.pair ? launch_by_dim<DT, QT, 16, 8>(L) : launch_by_dim<DT, QT, 8, 8>(L);
    case 16: return launch_by_dim<DT, QT, 16, 16>(L);
    case 32: return launch_by_dim<DT, QT, 32, 32>(L);
    }
    return cudaErrorNotSupported;
}

}  // namespace dec
}  // namespace pa
