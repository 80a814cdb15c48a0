// Prefill / chunked-prefill attention over the paged cache on the 5th-generation
// tensor cores ("01. PagedAttention 详解" §4, prefill: the new tokens' K, V
// are written through the block table first, then attention runs over the
// cache; the keys are gathered block by block through the table as in the
// decode loop of the same section).
//
// A query tile is 128 rows: TQ = 128 / G consecutive new tokens x the G query
// heads that share one kv head, so every K and V tile is loaded once for the
// whole group.  One CTA computes two adjacent query tiles (A and B) of one
// (sequence, kv head), so each K/V tile serves 256 rows and the two softmax
// warpgroups take turns with the tensor core.  Keys run in tiles of 128
// (128 / bs blocks, each fetched by its own tensor-map load from the block the
// table names).  Per key tile j and query tile X:
//
//   S_X = Q_X K_j^T       tcgen05.mma, M 128, N 128, K = D, A and B from shared
//                         memory, S in tensor memory
//   P_X = exp2(S_X * scale * log2 e - m)   softmax warpgroup X, one row per
//                         thread, causal + length mask; P is rounded to the
//                         operand type and written back over S_X in tensor memory
//   O_X += P_X V_j        tcgen05.mma, M 128, N = D, K 128, A (P) from tensor
//                         memory, B (V) from shared memory, O in tensor memory
//
// The running maximum m is raised only when a tile's maximum exceeds it by
// more than 8 (in log2 units); O and the running sum are then rescaled in
// place.  Between raises the probabilities stay below 2^8, so the result is
// the same softmax (the final division uses the same m for both sums).
//
// Warp roles (384 threads): warps 0-3 and 4-7 are the softmax and epilogue
// warpgroups of tiles A and B (warp w reads TMEM lanes 32(w%4)..32(w%4)+31,
// i.e. its 32 query rows); warp 8 loads (tensor-map copies of the two Q tiles
// once, then K and V tiles into rings); warp 9 allocates tensor memory, and
// one lane of warp 9 issues tile A's MMAs and one lane of warp 10 tile B's,
// each from its own scheduler (a tile's MMAs never queue behind the other
// tile's issue); warp 11 only completes the third warpgroup, whose registers
// go to the softmax warps.  The two softmax warps that share a scheduler (w
// and w + 4) take turns with their exponentials, so each has the special-
// function unit to itself, and a row's sum is taken after its P is handed to
// the MMA warp.  Tensor memory: S_A 0..127, O_A 128..255, S_B 256..383, O_B
// 384..511.  A tile's MMA lane issues its next S_X into the same columns right
// behind P_X.V (one thread's MMAs run in issue order), so the tensor core
// never idles waiting for P_X.V to finish.
// Every wait is bounded (2 s): on timeout the CTA records PA_DEV_WAIT_TIMEOUT
// with the wait's site, drains its own copies and MMAs, frees its tensor
// memory and exits.
//
// Prefix mode (shared-prefix decode, shared_prefix.cu): the query rows are the
// decode queries of all sequences, grid y is a chunk of the prefix every table
// shares, there is no causal mask, and the epilogue writes split-K records
// (m, l, o * v_scale) instead of normalised rows.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "tma_host.h"

namespace pf {

using namespace pa::dev;

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kPairGroup = 16;    // adjacent tile pairs scheduled side by side
constexpr int kSeg = 16384;       // 128 rows x 128 bytes: one operand segment
constexpr int kThreads = 384;     // 2 softmax warpgroups; a load warp, an MMA warp, 2 idle
// Register split (setmaxnreg): the kernel launches with 384 x 168 registers at
// most (three warps share each scheduler's 16K).  The softmax warpgroups take
// 208 each and the third warpgroup gives up to 64: 256 * 208 + 128 * 64 =
// 61440, which fits any launch allocation of 160 or more per thread.
constexpr int kRegsSoftmax = 208;
constexpr int kRegsOther = 64;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther <= kThreads * 160, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

struct Params {
    void* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;
    unsigned int* err;
    long long NB;
    int S, Hq, G, log2G, TQ, MB, bs, log2bs, max_qlen, n_pairs;
    float sl;                     // scale * log2(e) (* k_scale in prefix mode)
    // prefix mode (shared-prefix decode): the query rows are the S decode
    // queries, grid y is the prefix chunk, keys are chunk_tokens of the
    // prefix (row 0 of block_tables, or blocks 0.. of a converted copy when
    // identity_blocks), no causal mask, and the result is the split-K record
    // (m, l, o * v_scale) of partition `chunk` of every (sequence, head)
    int prefix, chunk_tokens, identity_blocks, max_parts;
    int pair_group;               // adjacent tile pairs per grid group (kPairGroup, or fewer)
    float2* ws_ml;
    float* ws_o;
    float v_scale;
};

template <int D>
struct Smem {
    static constexpr int NSEG = D / 64;             // 128-byte segments of a row
    static constexpr int ST = D == 64 ? 3 : 2;      // K and V ring depth
    static constexpr int TILE = NSEG * kSeg;        // 128 rows of D elements
    static constexpr int Q = 0;                     // query tiles A and B
    static constexpr int K = Q + 2 * TILE;
    static constexpr int V = K + ST * TILE;
    static constexpr int BAR = V + ST * TILE;
    // barriers: q, k_full[ST], k_free[ST], v_full[ST], v_free[ST], then per
    // query tile s_full, p_full, pv_done, o_full; drain; then per query tile
    // and softmax warp the turn of its exponentials
    static constexpr int NBAR = 1 + 4 * ST + 8 + 1 + 8 + 1;
    static constexpr int TMEM_SLOT = BAR + NBAR * 8;
    static constexpr int ABORT = TMEM_SLOT + 4;
    static constexpr int BYTES = ABORT + 4 + 1024;  // + slack to align the base to 1024
};

// ------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d_plain(uint32_t dst, const CUtensorMap* map,
                                                  uint32_t bar, int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2),
          "r"(c3)
        : "memory");
}

template <int N> __device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N> __device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(slot), "r"(cols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

// D (tensor memory, fp32) (+)= A (shared) x B (shared), kind::f16.  The
// shared-memory descriptors come as 32-bit halves: the issuing thread adds each
// K step's offset to the low word alone, one 32-bit add per descriptor
// (measured: +2.6 % per clock on the chunked-prefill workload against building
// every descriptor from its address).
__device__ __forceinline__ void tc_mma_lh(uint32_t d_tmem, uint32_t a_lo, uint32_t a_hi,
                                          uint32_t b_lo, uint32_t b_hi, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 da, db;\n\t"
        "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}"
        ::"r"(d_tmem), "r"(a_lo), "r"(a_hi), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D (tensor memory, fp32) (+)= A (tensor memory) x B (shared), kind::f16; the
// B descriptor as 32-bit halves.
__device__ __forceinline__ void tc_mma_ts_lh(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo,
                                             uint32_t b_hi, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 db;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
        " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),
          "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),
          "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
          "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
          "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// byte offset (between 64-element groups along M/N of an MN-major operand;
// unused for K-major), stride byte offset 1024 (between groups of 8 rows),
// the fixed descriptor version bit, and the swizzle mode.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B of one type
// (f16 = 0, bf16 = 1), A K-major, B K-major or MN-major, M 128, N.
__device__ __forceinline__ uint32_t idesc_f16(int ab_bf16, int b_mn_major, int N) {
    return (1u << 4) | ((uint32_t)ab_bf16 << 7) | ((uint32_t)ab_bf16 << 10) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

// 2^x on the special-function unit (ex2.approx.ftz: relative error about
// 2^-22, 2^-inf = +0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (a * b + c) on a pair of lanes in one instruction (fma.rn.f32x2).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// a + b on a pair of lanes in one instruction (add.rn.f32x2).
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

template <int DT> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<PA_BF16>(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
template <> __device__ __forceinline__ uint32_t pack2<PA_F16>(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
// Bounded wait by every lane of a warp; the outcome is warp-uniform.  A
// pipeline wait gives up early once another role has aborted the CTA; a drain
// wait (honor_abort false) does not, since it guards memory still in flight.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned int* err, unsigned site,
                                          bool honor_abort = true) {
    bool ok = mbar_try_wait(bar, parity);
    if (!__all_sync(~0u, ok)) {
        const uint64_t t0 = global_ns();
        while (!ok) {
#pragma unroll 1
            for (int i = 0; i < 64 && !ok; ++i) ok = mbar_try_wait(bar, parity);
            if (ok || (honor_abort && *abort_flag)) break;
            if (global_ns() - t0 > 2000000000ull) {
                atomicOr(err, PA_DEV_WAIT_TIMEOUT | (site << 16));
                break;
            }
        }
    }
    ok = __all_sync(~0u, ok);
    if (!ok) *abort_flag = 1;
    return ok;
}

// ------------------------------------------------------------------- kernel

template <int DT, int D>
__global__ void __launch_bounds__(kThreads, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, const Params p) {
    using L = Smem<D>;
    constexpr int NSEG = L::NSEG, ST = L::ST;
    // Launched as a programmatic dependent of the kernel before it: wait for
    // its memory (the cache append, or the prefix conversion) before reading.
    grid_dependency_wait();
    // Prefix mode: the suffix decode launched next reads the records only at
    // its very end (after its own griddepcontrol.wait), so let its CTAs start
    // on the SMs this grid leaves free.  Everything the kernels before this one
    // wrote is complete once the wait above returns (each of them waited for
    // its own predecessor), which the suffix decode relies on.
    if (p.prefix) launch_dependents();
    // grid (kPairGroup tile pairs x kv heads, sequences | prefix chunks, pair
    // groups): a group of adjacent tile pairs of one (sequence, kv head) runs
    // side by side and shares its K/V through L2, while groups run longest
    // first across all sequences (the causal tail stays short)
    const int PG = p.pair_group;
    const int g = (int)blockIdx.x / PG;
    const int pair = ((int)gridDim.z - 1 - (int)blockIdx.z) * PG + (PG - 1 - (int)blockIdx.x % PG);
    if (pair >= p.n_pairs) return;                        // past the last pair
    const bool pfx = p.prefix != 0;
    const int s = pfx ? 0 : (int)blockIdx.y;              // the sequence (table row)
    const int chunk = pfx ? (int)blockIdx.y : 0;          // prefix mode: the key chunk

    int q0 = 0, Ls = p.S, c = 0;
    if (!pfx) {
        q0 = p.query_start[s];
        Ls = p.query_start[s + 1] - q0;
        const int n = p.context_lens[s];
        if (Ls < 0 || Ls > n || Ls > p.max_qlen || (long long)n > (long long)p.MB * p.bs) {
            if (pair == 0 && g == 0 && threadIdx.x == 0) atomicOr(p.err, PA_DEV_BAD_CONTEXT);
            return;
        }
        c = n - Ls;                               // tokens cached before this chunk
    }
    const int TQ = p.TQ;
    const int iA = 2 * pair * TQ, iB = iA + TQ;   // first new token (row group) of tiles A and B
    if (iA >= Ls) return;                         // whole CTA: nothing to compute
    const bool hasB = iB < Ls;
    // keys each tile needs (causal: its last row's position + 1; prefix: the chunk)
    const int kvA = pfx ? p.chunk_tokens : c + min(Ls, iB);
    const int kvB = !hasB ? 0 : pfx ? p.chunk_tokens : c + min(Ls, iB + TQ);
    const int blk_base = pfx ? chunk * (p.chunk_tokens >> p.log2bs) : 0;
    const int ntA = (kvA + kBN - 1) / kBN;
    const int ntB = (kvB + kBN - 1) / kBN;
    const int kv_len = hasB ? kvB : kvA;
    const int nt = hasB ? ntB : ntA;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_addr(sm);
    const uint32_t sQ = sb + L::Q, sK = sb + L::K, sV = sb + L::V;
    const uint32_t bar0 = sb + L::BAR;
    const uint32_t q_full = bar0;
    auto k_full = [&](int i) { return bar0 + 8u * (1 + i); };
    auto k_free = [&](int i) { return bar0 + 8u * (1 + ST + i); };
    auto v_full = [&](int i) { return bar0 + 8u * (1 + 2 * ST + i); };
    auto v_free = [&](int i) { return bar0 + 8u * (1 + 3 * ST + i); };
    auto s_full = [&](int x) { return bar0 + 8u * (1 + 4 * ST + x); };
    auto p_full = [&](int x) { return bar0 + 8u * (3 + 4 * ST + x); };
    auto pv_done = [&](int x) { return bar0 + 8u * (5 + 4 * ST + x); };
    auto o_full = [&](int x) { return bar0 + 8u * (7 + 4 * ST + x); };
    const uint32_t drain = bar0 + 8u * (9 + 4 * ST);
    auto turn = [&](int x, int w) { return bar0 + 8u * (10 + 4 * ST + 4 * x + w); };
    const uint32_t v_zeroed = bar0 + 8u * (18 + 4 * ST);     // the last V tile's tail is zero
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        // with tile B, both MMA warps release every K and V stage
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full(i), 1);
            mbar_init(k_free(i), hasB ? 2 : 1);
            mbar_init(v_full(i), 1);
            mbar_init(v_free(i), hasB ? 2 : 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full(x), 1);
            mbar_init(p_full(x), 128);
            mbar_init(pv_done(x), 1);
            mbar_init(o_full(x), 1);
        }
        mbar_init(drain, hasB ? 2 : 1);
        for (int i = 0; i < 8; ++i) mbar_init(turn(i >> 2, i & 3), 1);
        mbar_init(v_zeroed, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(sb + L::TMEM_SLOT, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::TMEM_SLOT);
    auto tS = [&](int x) { return tmem + 256u * x; };          // scores, then P over them
    auto tO = [&](int x) { return tmem + 256u * x + 128u; };   // output accumulator

    if (warp == 8) {
        // ------------------------------------------------------------ loads
        regs_dec<kRegsOther>();
        const int bpt = kBN >> p.log2bs;                       // blocks per key tile
        const int need = (kv_len + p.bs - 1) >> p.log2bs;      // blocks the CTA reads
        const uint32_t box = (uint32_t)p.bs * 128u;
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, (hasB ? 2 : 1) * NSEG * kSeg);
            for (int x = 0; x < (hasB ? 2 : 1); ++x)
                for (int sg = 0; sg < NSEG; ++sg)
                    tma_load_3d(sQ + x * L::TILE + sg * kSeg, &tmq, q_full, sg * 64, g * p.G,
                                q0 + (x ? iB : iA));
        }
        int nk = 0, nvl = 0;                                   // K, V tiles started
        for (int j = 0; j < nt; ++j) {
            const int st = j % ST;
            const uint32_t par = ((j / ST) & 1) ^ 1;
            const int lb = j * bpt + lane;
            const bool want = lane < bpt && lb < need;
            int id = -1;
            if (want)
                id = p.identity_blocks ? blk_base + lb
                                       : p.block_tables[(size_t)s * p.MB + blk_base + lb];
            const bool valid = want && id >= 0 && (long long)id < p.NB;
            if (want && !valid) atomicOr(p.err, PA_DEV_BAD_BLOCK);
            const uint32_t bytes = (uint32_t)__popc(__ballot_sync(~0u, valid)) * NSEG * box;
            if (!warp_wait(k_free(st), par, abort_flag, p.err, 10)) break;
            if (lane == 0) mbar_arrive_expect_tx(k_full(st), bytes);
            __syncwarp();
            if (valid)
                for (int sg = 0; sg < NSEG; ++sg)
                    tma_load_4d_plain(sK + st * L::TILE + sg * kSeg + lane * box, &tmk, k_full(st),
                                      sg * 64, g, 0, id);
            nk = j + 1;
            if (!warp_wait(v_free(st), par, abort_flag, p.err, 11)) break;
            if (lane == 0) mbar_arrive_expect_tx(v_full(st), bytes);
            __syncwarp();
            if (valid)
                for (int sg = 0; sg < NSEG; ++sg)
                    tma_load_4d_plain(sV + st * L::TILE + sg * kSeg + lane * box, &tmv, v_full(st),
                                      sg * 64, g, 0, id);
            nvl = j + 1;
        }
        // every copy this warp started has landed before the CTA may exit
        // (immediate on the normal path, where the MMA warp consumed them all)
        for (int i = 0; i < ST; ++i) {
            // the last tile started in slot i is the largest j < count with j % ST == i
            if (nk > i) {
                const int jl = i + (nk - 1 - i) / ST * ST;
                warp_wait(k_full(i), (jl / ST) & 1, abort_flag, p.err, 17, false);
            }
            if (nvl > i) {
                const int jl = i + (nvl - 1 - i) / ST * ST;
                warp_wait(v_full(i), (jl / ST) & 1, abort_flag, p.err, 17, false);
            }
        }
        warp_wait(q_full, 0, abort_flag, p.err, 17, false);
    } else if (warp == 9 || (warp == 10 && hasB)) {
        // ------------------------------------------------------------- MMAs
        // Warp 9 issues tile A's MMAs and warp 10 tile B's, each from its own
        // scheduler, so a tile's P.V and next S go out as soon as its P is
        // handed over rather than behind the other tile's.  With tile B both
        // warps release every K and V stage (the free barriers count two); a
        // warp whose tile needs fewer key tiles arrives on the stages it does
        // not read once they are filled, so both warps' arrivals on a barrier
        // are always for the same use of the stage.
        regs_dec<kRegsOther>();
        const int x = warp - 9;
        const int ntx = x ? ntB : ntA;
        // the pair's last key tile (read by B, and by A when ntA == nt): the
        // warp of the tile that reads it last zeroes its V tail
        const bool zeroes = hasB ? x == 1 : true;
        constexpr int ABF = DT == PA_BF16 ? 1 : 0;
        const uint32_t id_s = idesc_f16(ABF, 0, kBN);
        const uint32_t id_o = idesc_f16(ABF, 1, D);
        // S_X = Q_X K^T for key tile j (K in ring slot st)
        auto issue_s = [&](int st) {
            tc_fence_after();
            if (lane == 0) {
                const uint32_t kb = sK + st * L::TILE, qb = sQ + x * L::TILE;
                // low word: start address / 16 (14 bits, no carry below 2^18
                // bytes) | leading offset 16 B << 16; high word constant
                const uint32_t hi = (uint32_t)(sdesc(0, 16) >> 32);
                const uint32_t alo = (qb >> 4) | (1u << 16), blo = (kb >> 4) | (1u << 16);
                const uint32_t d = tS(x);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kSeg + (kk & 3) * 32) >> 4;
                    tc_mma_lh(d, alo + off, hi, blo + off, hi, id_s, kk > 0);
                }
                tc_commit(s_full(x));
                tc_commit(k_free(st));
            }
            __syncwarp();
        };
        bool ok = warp_wait(q_full, 0, abort_flag, p.err, 7) &&
                  warp_wait(k_full(0), 0, abort_flag, p.err, 8);
        if (ok) issue_s(0);
        for (int j = 0; j < nt && ok; ++j) {
            const int st = j % ST, st1 = (j + 1) % ST;
            if (!(ok = warp_wait(v_full(st), (j / ST) & 1, abort_flag, p.err, 9))) break;
            const uint32_t vb = sV + st * L::TILE;
            if (j == nt - 1 && zeroes) {
                // Rows at or past kv_len hold another token's values, the cache's
                // unused tail slots or stale tiles: zero them, since a zero
                // probability times a NaN would still poison the product.
                const int z0 = kv_len - j * kBN;
                const int chunks = (kBN - z0) * 8;              // 16-byte chunks per segment
                for (int sg = 0; sg < NSEG; ++sg)
                    for (int xx = lane; xx < chunks; xx += 32)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};"
                                     ::"r"(vb + sg * kSeg + z0 * 128 + xx * 16), "r"(0) : "memory");
                fence_proxy_async_smem();
                __syncwarp();
                if (hasB && ntA == nt && lane == 0) mbar_arrive(v_zeroed);
                __syncwarp();
            } else if (j == nt - 1 && j < ntx) {
                if (!(ok = warp_wait(v_zeroed, 0, abort_flag, p.err, 9))) break;
            }
            if (j < ntx) {
                if (!(ok = warp_wait(p_full(x), j & 1, abort_flag, p.err, 13))) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t vhi = (uint32_t)(sdesc(0, kSeg) >> 32);
                    const uint32_t vlo = (vb >> 4) | ((uint32_t)(kSeg >> 4) << 16);
                    const uint32_t to = tO(x), ts = tS(x);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        tc_mma_ts_lh(to, ts + kk * 8, vlo + kk * 128, vhi, id_o,
                                     (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(pv_done(x));
                    if (j == ntx - 1) tc_commit(o_full(x));
                    tc_commit(v_free(st));
                }
            } else if (lane == 0) {
                mbar_arrive(v_free(st));                       // this tile does not read tile j
            }
            __syncwarp();
            if (j + 1 < nt) {
                // The next scores overwrite P_X in the same columns.  They are
                // issued right behind P_X.V: the MMAs one thread issues run in
                // issue order, so P_X.V has read P_X before S_X(j+1) is written.
                if (!(ok = warp_wait(k_full(st1), ((j + 1) / ST) & 1, abort_flag, p.err, 8))) break;
                if (j + 1 < ntx) {
                    issue_s(st1);
                } else {
                    if (lane == 0) mbar_arrive(k_free(st1));
                    __syncwarp();
                }
            }
        }
        // every MMA this warp issued completes before tensor memory is freed
        if (lane == 0) tc_commit(drain);
        __syncwarp();
        warp_wait(drain, 0, abort_flag, p.err, 16, false);
    } else if (warp >= 10) {
        regs_dec<kRegsOther>();
    } else if (warp < 4 || hasB) {
        // ---------------------------------------- softmax (rows of tile X)
        regs_inc<kRegsSoftmax>();
        const int x = warp >> 2;
        const int r = threadIdx.x & 127;                     // row = TMEM lane
        const int iX = x ? iB : iA;
        const int kvX = x ? kvB : kvA;
        const int ntx = x ? ntB : ntA;
        const int it = iX + (r >> p.log2G);                  // new-token index of the row
        const bool row_ok = it < Ls;
        const int limit = row_ok && !pfx ? c + it + 1 : kvX;  // keys 0..limit-1 are visible
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        const float sl = p.sl;
        const uint32_t my_turn = turn(x, warp & 3), next_turn = turn(x ^ 1, warp & 3);
        float m_use = -INFINITY, lsum = 0.f;
        bool ok = true;
        for (int j = 0; j < ntx; ++j) {
            if (!(ok = warp_wait(s_full(x), j & 1, abort_flag, p.err, 12))) break;
            tc_fence_after();
            float sv[kBN];
#pragma unroll
            for (int c4 = 0; c4 < kBN / 32; ++c4) tmem_ld32(tS(x) + lrow + c4 * 32, sv + c4 * 32);
            tmem_wait_ld();
            // keys past a row's position (causal bound, or past the tile's last
            // needed key) become -inf; a tile no row masks skips the compares
            if ((j + 1) * kBN > (pfx ? kvX : c + iX + 1)) {
                const int nv = limit - j * kBN;
#pragma unroll
                for (int k = 0; k < kBN; ++k)
                    if (k >= nv) sv[k] = -INFINITY;
            }
            // row maximum as 8 independent chains of three-input maxima (a
            // single chain of dependent maxima would sit on the critical path)
            float pm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pm[i] = sv[i];
#pragma unroll
            for (int k = 8; k < kBN; k += 2) pm[(k >> 1) & 7] = max3(pm[(k >> 1) & 7], sv[k], sv[k + 1]);
            const float tmax = fmaxf(max3(pm[0], pm[1], pm[2]),
                                     fmaxf(max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            const float m_new = fmaxf(m_use, tmax * sl);       // scale > 0
            const bool raise = m_new > m_use + kRescaleLog2;
            const float alpha = raise ? ex2(m_use - m_new) : 1.f;
            if (raise) m_use = m_new;
            lsum *= alpha;
            if (j > 0 && __any_sync(~0u, raise)) {
                // O_X holds P.V of tiles 0..j-1 once the last of them completes
                if (!(ok = warp_wait(pv_done(x), (j - 1) & 1, abort_flag, p.err, 14))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    float o[32];
                    tmem_ld32(tO(x) + lrow + c4 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(tO(x) + lrow + c4 * 32, o);
                }
                tmem_wait_st();
            }
            // The two softmax warps of one scheduler (warp w of tile A, warp
            // w + 4 of tile B) take turns with their exponentials, A(j), B(j),
            // A(j + 1) ..., so each runs with the special-function unit to
            // itself instead of both at half speed; B's tiles past A's last
            // one need no turn.
            if (hasB && (x ? j < ntA : j > 0) &&
                !(ok = warp_wait(my_turn, (j - 1 + x) & 1, abort_flag, p.err, 18)))
                break;
            // probabilities, rounded to the operand type, two per 32-bit
            // column over the scores they came from (the A operand of P.V);
            // pairs of scores share one packed FMA
            const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
            for (int c16 = 0; c16 < kBN / 32; ++c16) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = c16 * 32 + 2 * e;
                    const float2 xy = fma2(make_float2(sv[k], sv[k + 1]), sl2, nm2);
                    sv[k] = ex2(xy.x);
                    sv[k + 1] = ex2(xy.y);
                    w[e] = pack2<DT>(sv[k], sv[k + 1]);
                }
                tmem_st16(tS(x) + lrow + c16 * 16, w);
            }
            if (hasB && (x == 0 || j + 1 < ntA)) {
                __syncwarp();
                if (lane == 0) mbar_arrive(next_turn);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(p_full(x));
            // the row sum is not on the way to P.V: it is taken after the hand-off
            float2 ps[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int k = 0; k < kBN; k += 2)
                ps[(k >> 1) & 3] = add2(ps[(k >> 1) & 3], make_float2(sv[k], sv[k + 1]));
            lsum += ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) +
                    ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
        }
        if (ok) ok = warp_wait(o_full(x), 0, abort_flag, p.err, 15);
        if (ok && pfx) {
            // the split-K record of partition `chunk`: running maximum (log2
            // units), sum, and the unnormalised sum of weighted values
            tc_fence_after();
            const int h = g * p.G + (r & (p.G - 1));
            const size_t row = ((size_t)it * p.Hq + h) * p.max_parts + chunk;
            float* dst = p.ws_o + row * D;
#pragma unroll 1
            for (int c4 = 0; c4 < D / 32; ++c4) {
                float o[32];
                tmem_ld32(tO(x) + lrow + c4 * 32, o);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        reinterpret_cast<float4*>(dst + c4 * 32)[v] =
                            make_float4(o[4 * v] * p.v_scale, o[4 * v + 1] * p.v_scale,
                                        o[4 * v + 2] * p.v_scale, o[4 * v + 3] * p.v_scale);
                }
            }
            if (row_ok) p.ws_ml[row] = make_float2(m_use, lsum);
        } else if (ok) {
            tc_fence_after();
            const float inv = 1.f / lsum;
            const int h = g * p.G + (r & (p.G - 1));
            uint8_t* orow = static_cast<uint8_t*>(p.out) +
                            ((size_t)(q0 + it) * p.Hq + h) * (size_t)D * 2;
#pragma unroll 1
            for (int c4 = 0; c4 < D / 32; ++c4) {
                float o[32];
                tmem_ld32(tO(x) + lrow + c4 * 32, o);
                tmem_wait_ld();
                if (row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 64);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack2<DT>(o[8 * v + 0] * inv, o[8 * v + 1] * inv);
                        w.y = pack2<DT>(o[8 * v + 2] * inv, o[8 * v + 3] * inv);
                        w.z = pack2<DT>(o[8 * v + 4] * inv, o[8 * v + 5] * inv);
                        w.w = pack2<DT>(o[8 * v + 6] * inv, o[8 * v + 7] * inv);
                        dst[v] = w;
                    }
                }
            }
        }
        tc_fence_before();
    } else {
        regs_inc<kRegsSoftmax>();      // tile B is empty: the warpgroup still takes its share
    }

    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int DT, int D>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const Params& p, dim3 grid, cudaStream_t st) {
    const cudaError_t attr = pa::dev::ensure_dynamic_smem<prefill_kernel<DT, D>>(Smem<D>::BYTES);
    if (attr != cudaSuccess) return attr;
    return launch_pdl(prefill_kernel<DT, D>, grid, dim3(kThreads), (size_t)Smem<D>::BYTES, st, mq,
                      mk, mv, p);
}

// ------------------------------------------------- CTA-pair kernel (D = 128)
// The same attention with the two query tiles of a pair on two SMs, one per
// CTA of a cluster of two, and the tensor-core instructions of the pair
// (cta_group::2): one MMA of M = 256 rows computes both tiles' scores (each CTA
// holds its tile's 128 query rows and half the key tile, 64 keys; each SM's
// tensor memory receives its tile's 128 rows of all 128 keys), and one of
// M = 256 adds P.V (each CTA holds half the value tile, 64 dims of 128 keys,
// and its tile's P in its own tensor memory).  Each SM thus loads half of every
// K and V tile, and its tensor memory holds two score buffers and O
// (S_0 0..127, S_1 128..255, O 256..383): the scores of key tile j + 1 are
// computed while the softmax works on tile j, so the softmax warpgroup of each
// SM runs its tiles back to back instead of waiting for P.V and the next S
// after every tile.  The leader CTA (cluster rank 0, tile A) issues every MMA
// from one thread and commits each to both CTAs' barriers; each CTA's copies
// land in its own shared memory and complete on the leader's barriers, except
// the last V tile, whose rows past the tile's keys each CTA zeroes itself
// before it signals the leader.  192 threads: warps 0-3 the softmax (one query
// row per thread), warp 4 the copies, warp 5 tensor memory and (leader) the
// MMAs.  Chunked prefill and prefill only (no prefix mode).
constexpr int kThreads2 = 192;

struct Smem2 {
    static constexpr int ST = 3;                        // K and V ring depth
    static constexpr int KSEG = kSeg / 2;               // 64 key rows x 128 bytes
    static constexpr int KH = 2 * KSEG;                 // this CTA's 64 keys x 128 dims
    static constexpr int VH = kSeg;                     // 128 keys x this CTA's 64 dims
    static constexpr int Q = 0;                         // this CTA's 128 query rows, 2 segments
    static constexpr int K = Q + 2 * kSeg;
    static constexpr int V = K + ST * KH;
    static constexpr int BAR = V + ST * VH;
    // q_full, k_full[ST], v_full[ST] (leader: both CTAs' copies), k_free[ST],
    // v_free[ST] (each CTA: the pair's MMAs are done with the slot), s_full[2],
    // p_full[2] (leader: the 8 softmax warps), pv_done, o_full, drain (leader),
    // v_last (leader: both CTAs' last V tile zeroed past the keys), v_mine
    static constexpr int NBAR = 1 + 4 * ST + 2 + 2 + 1 + 1 + 1 + 1 + 1;
    static constexpr int TMEM_SLOT = BAR + NBAR * 8;
    static constexpr int ABORT = TMEM_SLOT + 4;
    static constexpr int BYTES = ABORT + 4 + 1024;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// The shared::cluster address of `local` in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local), "r"(rank));
    return a;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// Arrive on an mbarrier of a CTA of the cluster.  What it orders is tensor
// memory (tcgen05.wait::st and fence::before_thread_sync before it) and this
// CTA's shared memory ahead of the peer's bulk copies, not generic memory
// the other CTA reads, so it takes the default semantics rather than a
// cluster-scope release (whose fence stalled the softmax warps).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t slot, uint32_t cols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(slot), "r"(cols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t cols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}
// The completion of this thread's earlier tcgen05 operations, on the mbarrier
// at `bar`'s offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(bar), "h"((uint16_t)3) : "memory");
}
// ... on this CTA's mbarrier only.
__device__ __forceinline__ void tc_commit_local2(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_mma2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_mma_ts2(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Tensor-map copies into this CTA's shared memory that complete on an
// mbarrier of the pair's leader (`bar` a shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2),
          "r"(c3)
        : "memory");
}
// Instruction descriptor of kind::f16 for the pair: M 256 (128 rows per CTA).
__device__ __forceinline__ uint32_t idesc2_f16(int ab_bf16, int b_mn_major, int N) {
    return (1u << 4) | ((uint32_t)ab_bf16 << 7) | ((uint32_t)ab_bf16 << 10) |
           ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

template <int DT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads2, 1)
prefill2_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const Params p) {
    using L = Smem2;
    constexpr int D = 128, ST = L::ST;
    grid_dependency_wait();
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    // grid (2 x kPairGroup pairs x kv heads, sequences, pair groups); the two
    // CTAs of a cluster are the tiles A and B of one pair, and take every early
    // exit together (their conditions depend on the pair and sequence only)
    const int PG = p.pair_group;
    const int unit = (int)blockIdx.x >> 1;
    const int g = unit / PG;
    const int pair = ((int)gridDim.z - 1 - (int)blockIdx.z) * PG + (PG - 1 - unit % PG);
    if (pair >= p.n_pairs) return;
    const int s = (int)blockIdx.y;
    const int q0 = p.query_start[s];
    const int Ls = p.query_start[s + 1] - q0;
    const int n = p.context_lens[s];
    if (Ls < 0 || Ls > n || Ls > p.max_qlen || (long long)n > (long long)p.MB * p.bs) {
        if (leader && pair == 0 && g == 0 && threadIdx.x == 0) atomicOr(p.err, PA_DEV_BAD_CONTEXT);
        return;
    }
    const int c = n - Ls;
    const int TQ = p.TQ;
    const int iA = 2 * pair * TQ, iB = iA + TQ;
    if (iA >= Ls) return;
    const bool hasB = iB < Ls;
    const int kvA = c + min(Ls, iB);
    const int kv_len = hasB ? c + min(Ls, iB + TQ) : kvA;     // keys the pair reads
    const int nt = (kv_len + kBN - 1) / kBN;
    const int iX = leader ? iA : iB;                          // this CTA's first new token

    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    const uint32_t sb = smem_addr(sm);
    const uint32_t sQ = sb + L::Q, sK = sb + L::K, sV = sb + L::V;
    const uint32_t bar0 = sb + L::BAR;
    const uint32_t q_full = bar0;
    auto k_full = [&](int i) { return bar0 + 8u * (1 + i); };
    auto v_full = [&](int i) { return bar0 + 8u * (1 + ST + i); };
    auto k_free = [&](int i) { return bar0 + 8u * (1 + 2 * ST + i); };
    auto v_free = [&](int i) { return bar0 + 8u * (1 + 3 * ST + i); };
    auto s_full = [&](int b) { return bar0 + 8u * (1 + 4 * ST + b); };
    auto p_full = [&](int b) { return bar0 + 8u * (3 + 4 * ST + b); };
    const uint32_t pv_done = bar0 + 8u * (5 + 4 * ST);
    const uint32_t o_full = bar0 + 8u * (6 + 4 * ST);
    const uint32_t drain = bar0 + 8u * (7 + 4 * ST);
    const uint32_t v_last = bar0 + 8u * (8 + 4 * ST);
    const uint32_t v_mine = bar0 + 8u * (9 + 4 * ST);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < ST; ++i) {
            mbar_init(k_full(i), 1);
            mbar_init(v_full(i), 1);
            mbar_init(k_free(i), 1);
            mbar_init(v_free(i), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(s_full(b), 1);
            mbar_init(p_full(b), 8);
        }
        mbar_init(pv_done, 1);
        mbar_init(o_full, 1);
        mbar_init(drain, 1);
        mbar_init(v_last, 2);
        mbar_init(v_mine, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc2(sb + L::TMEM_SLOT, kTmemCols);
        tmem_relinquish2();
    }
    // both CTAs' barriers and tensor memory exist before either touches the other's
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sm + L::TMEM_SLOT);
    auto tS = [&](int b) { return tmem + 128u * b; };        // scores, then P over them
    const uint32_t tO = tmem + 256u;                           // output accumulator

    if (warp == 4) {
        // ------------------------------------------------------------ loads
        const int bpt = kBN >> p.log2bs;                       // blocks per key tile
        const int half = bpt >> 1;                             // blocks of this CTA's K half
        const int need = (kv_len + p.bs - 1) >> p.log2bs;
        const uint32_t box = (uint32_t)p.bs * 128u;
        const uint32_t lq = cluster_addr(q_full, 0);
        if (lane == 0) {
            if (leader) mbar_arrive_expect_tx(q_full, 2 * 2 * kSeg);
            for (int sg = 0; sg < 2; ++sg)
                tma_load_3d_pair(sQ + sg * kSeg, &tmq, lq, sg * 64, g * p.G, q0 + iX);
        }
        int nk = 0;
        for (int j = 0; j < nt; ++j) {
            const int st = j % ST;
            const uint32_t par = ((j / ST) & 1) ^ 1;
            const int lb = j * bpt + lane;
            const bool want = lane < bpt && lb < need;
            int id = -1;
            if (want) id = p.block_tables[(size_t)s * p.MB + lb];
            const bool valid = want && id >= 0 && (long long)id < p.NB;
            if (leader && want && !valid) atomicOr(p.err, PA_DEV_BAD_BLOCK);
            const uint32_t nvalid = (uint32_t)__popc(__ballot_sync(~0u, valid));
            // K: this CTA's half of the tile's blocks, two 64-dim segments each
            if (!warp_wait(k_free(st), par, abort_flag, p.err, 10)) break;
            if (leader && lane == 0) mbar_arrive_expect_tx(k_full(st), nvalid * 2 * box);
            __syncwarp();
            if (valid && lane / half == (int)rank)
                for (int sg = 0; sg < 2; ++sg)
                    tma_load_4d_pair(sK + st * L::KH + sg * L::KSEG + (lane - (int)rank * half) * box,
                                     &tmk, cluster_addr(k_full(st), 0), sg * 64, g, 0, id);
            nk = j + 1;
            // V: this CTA's 64 dims of every block of the tile
            if (!warp_wait(v_free(st), par, abort_flag, p.err, 11)) break;
            if (j + 1 < nt) {
                if (leader && lane == 0) mbar_arrive_expect_tx(v_full(st), nvalid * 2 * box);
                __syncwarp();
                if (valid)
                    tma_load_4d_pair(sV + st * L::VH + lane * box, &tmv, cluster_addr(v_full(st), 0),
                                     (int)rank * 64, g, 0, id);
            } else {
                // The last tile lands on this CTA's own barrier: its rows at or
                // past the pair's keys hold another token's values, the cache's
                // unused tail slots or stale tiles, and are zeroed here (a zero
                // probability times a NaN would still poison the product).
                if (lane == 0) mbar_arrive_expect_tx(v_mine, nvalid * box);
                __syncwarp();
                if (valid)
                    tma_load_4d_plain(sV + st * L::VH + lane * box, &tmv, v_mine, (int)rank * 64, g,
                                      0, id);
                if (!warp_wait(v_mine, 0, abort_flag, p.err, 9, false)) break;
                const int z0 = kv_len - j * kBN;
                for (int xx = lane; xx < (kBN - z0) * 8; xx += 32)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};"
                                 ::"r"(sV + st * L::VH + z0 * 128 + xx * 16), "r"(0) : "memory");
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (leader) mbar_arrive(v_last);
                    else mbar_arrive_cluster(cluster_addr(v_last, 0));
                }
            }
        }
        // (leader) every copy of the pair has landed before the CTAs may exit:
        // immediate on the normal path, where the MMAs consumed them all
        if (leader)
            for (int i = 0; i < ST && i < nk; ++i) {
                const int jl = i + (nk - 1 - i) / ST * ST;
                warp_wait(k_full(i), (jl / ST) & 1, abort_flag, p.err, 17, false);
                if (jl + 1 < nt) warp_wait(v_full(i), (jl / ST) & 1, abort_flag, p.err, 17, false);
            }
        if (leader) warp_wait(q_full, 0, abort_flag, p.err, 17, false);
    } else if (warp == 5) {
        // ------------------------------------------------ MMAs (leader only)
        if (leader) {
            constexpr int ABF = DT == PA_BF16 ? 1 : 0;
            const uint32_t id_s = idesc2_f16(ABF, 0, kBN);
            const uint32_t id_o = idesc2_f16(ABF, 1, D);
            // S_b = Q K_j^T, both tiles: K_j's halves in both CTAs' ring slot st
            auto issue_s = [&](int b, int st) {
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kb = sK + st * L::KH;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        tc_mma2(tS(b), sdesc(sQ + (kk >> 2) * kSeg + (kk & 3) * 32, 16),
                                sdesc(kb + (kk >> 2) * L::KSEG + (kk & 3) * 32, 16), id_s, kk > 0);
                    }
                    tc_commit_pair(s_full(b));
                    tc_commit_pair(k_free(st));
                }
                __syncwarp();
            };
            bool ok = warp_wait(q_full, 0, abort_flag, p.err, 7) &&
                      warp_wait(k_full(0), 0, abort_flag, p.err, 8);
            if (ok) issue_s(0, 0);
            if (ok && nt > 1 && (ok = warp_wait(k_full(1 % ST), (1 / ST) & 1, abort_flag, p.err, 8)))
                issue_s(1, 1 % ST);
            for (int j = 0; j < nt && ok; ++j) {
                const int st = j % ST, b = j & 1;
                if (!(ok = warp_wait(p_full(b), (j >> 1) & 1, abort_flag, p.err, 13))) break;
                if (!(ok = j + 1 < nt ? warp_wait(v_full(st), (j / ST) & 1, abort_flag, p.err, 9)
                                      : warp_wait(v_last, 0, abort_flag, p.err, 9)))
                    break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t vb = sV + st * L::VH;
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        tc_mma_ts2(tO, tS(b) + kk * 8, sdesc(vb + kk * 16 * 128, kSeg), id_o,
                                   (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit_pair(pv_done);
                    tc_commit_pair(v_free(st));
                    if (j == nt - 1) tc_commit_pair(o_full);
                }
                __syncwarp();
                if (j + 2 < nt) {
                    // S_b(j + 2) overwrites P_b(j): issued behind P_b(j).V, and one
                    // thread's MMAs execute in issue order
                    const int st2 = (j + 2) % ST;
                    if (!(ok = warp_wait(k_full(st2), ((j + 2) / ST) & 1, abort_flag, p.err, 8)))
                        break;
                    issue_s(b, st2);
                }
            }
            if (lane == 0) tc_commit_local2(drain);
            __syncwarp();
            warp_wait(drain, 0, abort_flag, p.err, 16, false);
        }
    } else {
        // ------------------------------------------------ softmax (4 warps)
        const int r = threadIdx.x;                           // row = tensor-memory lane
        const int it = iX + (r >> p.log2G);                  // new-token index of the row
        const bool row_ok = it < Ls;
        const int limit = row_ok ? c + it + 1 : kv_len;      // keys 0..limit-1 are visible
        const uint32_t lrow = (uint32_t)(warp * 32) << 16;
        const float sl = p.sl;
        const uint32_t my_p_full0 = leader ? p_full(0) : cluster_addr(p_full(0), 0);
        const uint32_t my_p_full1 = leader ? p_full(1) : cluster_addr(p_full(1), 0);
        float m_use = -INFINITY, lsum = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            const int b = j & 1;
            if (!(ok = warp_wait(s_full(b), (j >> 1) & 1, abort_flag, p.err, 12))) break;
            tc_fence_after();
            float sv[kBN];
#pragma unroll
            for (int c4 = 0; c4 < kBN / 32; ++c4) tmem_ld32(tS(b) + lrow + c4 * 32, sv + c4 * 32);
            tmem_wait_ld();
            if ((j + 1) * kBN > c + iX + 1) {
                const int nv = limit - j * kBN;
#pragma unroll
                for (int k = 0; k < kBN; ++k)
                    if (k >= nv) sv[k] = -INFINITY;
            }
            float pm[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pm[i] = sv[i];
#pragma unroll
            for (int k = 8; k < kBN; k += 2) pm[(k >> 1) & 7] = max3(pm[(k >> 1) & 7], sv[k], sv[k + 1]);
            const float tmax = fmaxf(max3(pm[0], pm[1], pm[2]),
                                     fmaxf(max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])));
            const float m_new = fmaxf(m_use, tmax * sl);
            const bool raise = m_new > m_use + kRescaleLog2;
            const float alpha = raise ? ex2(m_use - m_new) : 1.f;
            if (raise) m_use = m_new;
            lsum *= alpha;
            if (j > 0 && __any_sync(~0u, raise)) {
                // O holds P.V of tiles 0..j-1 once the last of them completes
                if (!(ok = warp_wait(pv_done, (j - 1) & 1, abort_flag, p.err, 14))) break;
                tc_fence_after();
#pragma unroll 1
                for (int c4 = 0; c4 < D / 32; ++c4) {
                    float o[32];
                    tmem_ld32(tO + lrow + c4 * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= alpha;
                    tmem_st32(tO + lrow + c4 * 32, o);
                }
                tmem_wait_st();
            }
            const float2 sl2 = make_float2(sl, sl), nm2 = make_float2(-m_use, -m_use);
#pragma unroll
            for (int c16 = 0; c16 < kBN / 32; ++c16) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int k = c16 * 32 + 2 * e;
                    const float2 xy = fma2(make_float2(sv[k], sv[k + 1]), sl2, nm2);
                    sv[k] = ex2(xy.x);
                    sv[k + 1] = ex2(xy.y);
                    w[e] = pack2<DT>(sv[k], sv[k + 1]);
                }
                tmem_st16(tS(b) + lrow + c16 * 16, w);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(p_full(b));
                else mbar_arrive_cluster(b ? my_p_full1 : my_p_full0);
            }
            float2 ps[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int k = 0; k < kBN; k += 2)
                ps[(k >> 1) & 3] = add2(ps[(k >> 1) & 3], make_float2(sv[k], sv[k + 1]));
            lsum += ((ps[0].x + ps[0].y) + (ps[1].x + ps[1].y)) +
                    ((ps[2].x + ps[2].y) + (ps[3].x + ps[3].y));
        }
        if (ok) ok = warp_wait(o_full, 0, abort_flag, p.err, 15);
        if (ok) {
            tc_fence_after();
            const float inv = 1.f / lsum;
            const int h = g * p.G + (r & (p.G - 1));
            uint8_t* orow = static_cast<uint8_t*>(p.out) + ((size_t)(q0 + it) * p.Hq + h) * (size_t)D * 2;
#pragma unroll 1
            for (int c4 = 0; c4 < D / 32; ++c4) {
                float o[32];
                tmem_ld32(tO + lrow + c4 * 32, o);
                tmem_wait_ld();
                if (row_ok) {
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) w[e] = pack2<DT>(o[2 * e] * inv, o[2 * e + 1] * inv);
#pragma unroll
                    for (int v = 0; v < 4; ++v)
                        reinterpret_cast<uint4*>(orow + c4 * 64)[v] =
                            make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
                }
            }
        }
    }
    // Every MMA of the pair has completed (the leader drained them) and no lane
    // of either CTA reads tensor memory any more: free it, in both CTAs.
    tc_fence_before();
    cluster_sync();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc2(tmem, kTmemCols);
    }
}

template <int DT>
cudaError_t launch2(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const Params& p, dim3 grid, cudaStream_t st) {
    const cudaError_t attr = pa::dev::ensure_dynamic_smem<prefill2_kernel<DT>>(Smem2::BYTES);
    if (attr != cudaSuccess) return attr;
    return launch_pdl(prefill2_kernel<DT>, grid, dim3(kThreads2), (size_t)Smem2::BYTES, st, mq, mk,
                      mv, p);
}

}  // namespace pf

using pa::fail;

// Shared-prefix decode, step 1 (declared in pa_internal.h): the split-K
// records of the prefix partitions of every (sequence, head), from one pass
// of the tensor-core kernel in prefix mode.
pa_status pa::prefix_records(const void* q, pa_dtype dt, const void* k_src, const void* v_src,
                             int64_t src_blocks, const int32_t* table_row0, int S, int Hq,
                             int Hkv, int D, int bs, int prefix_tokens, int chunk_tokens,
                             float sl, float v_scale, float2* ws_ml, float* ws_o, int max_parts,
                             pa_stream_t stream) {
    const int G = Hq / Hkv;
    const int TQ = pf::kBM / G;
    const long long n_qt = ((long long)S + TQ - 1) / TQ;
    const long long n_pairs = (n_qt + 1) / 2;
    const int chunks = prefix_tokens / chunk_tokens;
    if (n_pairs > 65535 || chunks > 65535 || Hkv > 65535)
        return fail(PA_ERR_UNSUPPORTED, "prefix grid too large");
    CUtensorMap mq, mk, mv;
    pa_status st = pa::make_rows_map(&mq, q, dt, S, Hq, D, G, TQ);
    if (st) return st;
    st = pa::make_cache_map(&mk, k_src, dt, src_blocks, bs, Hkv, D);
    if (st) return st;
    st = pa::make_cache_map(&mv, v_src, dt, src_blocks, bs, Hkv, D);
    if (st) return st;
    unsigned int* err = pa::device_error_word();
    if (!err) return PA_ERR_CUDA;
    pf::Params p = {};
    p.block_tables = table_row0;
    p.err = err;
    p.NB = src_blocks;
    p.S = S;
    p.Hq = Hq;
    p.G = G;
    p.log2G = __builtin_ctz((unsigned)G);
    p.TQ = TQ;
    p.MB = 0;
    p.bs = bs;
    p.log2bs = __builtin_ctz((unsigned)bs);
    p.max_qlen = S;
    p.n_pairs = (int)n_pairs;
    p.sl = sl;
    p.prefix = 1;
    p.chunk_tokens = chunk_tokens;
    p.identity_blocks = table_row0 ? 0 : 1;
    p.max_parts = max_parts;
    p.ws_ml = ws_ml;
    p.ws_o = ws_o;
    p.v_scale = v_scale;
    // as many pair slots per group as there are pairs (no CTA that only exits:
    // each would hold a whole SM's shared memory for a moment)
    p.pair_group = (int)(n_pairs < pf::kPairGroup ? n_pairs : pf::kPairGroup);
    const dim3 grid((unsigned)(Hkv * p.pair_group), (unsigned)chunks,
                    (unsigned)((n_pairs + p.pair_group - 1) / p.pair_group));
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == PA_BF16)
        e = D == 64 ? pf::launch<PA_BF16, 64>(mq, mk, mv, p, grid, cs)
                    : pf::launch<PA_BF16, 128>(mq, mk, mv, p, grid, cs);
    else
        e = D == 64 ? pf::launch<PA_F16, 64>(mq, mk, mv, p, grid, cs)
                    : pf::launch<PA_F16, 128>(mq, mk, mv, p, grid, cs);
    if (e != cudaSuccess) return pa::cuda_fail(e, "prefix kernel launch");
    return PA_OK;
}

extern "C" pa_status pa_prefill(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                                const void* value_cache, pa_dtype cache_dt,
                                const int32_t* block_tables, int MB, const int32_t* context_lens,
                                const int32_t* query_start, int S, int T, int Hq, int Hkv, int D,
                                int bs, int64_t NB, int max_query_len, float scale,
                                pa_stream_t stream) {
    PA_NVTX_RANGE("pa_prefill");
    pa::clear_error();
    if (!pa::valid_dtype(q_dt) || !pa::valid_dtype(cache_dt))
        return fail(PA_ERR_INVALID_ARG, "unknown dtype");
    if (q_dt != cache_dt || (q_dt != PA_F16 && q_dt != PA_BF16))
        return fail(PA_ERR_UNSUPPORTED, "prefill takes q and cache both f16 or both bf16");
    if (D != 64 && D != 128) return fail(PA_ERR_UNSUPPORTED, "head size %d (64 or 128)", D);
    if (bs != 8 && bs != 16 && bs != 32) return fail(PA_ERR_UNSUPPORTED, "block size %d", bs);
    if (S < 0 || T < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || MB <= 0 || NB <= 0 ||
        max_query_len < 0)
        return fail(PA_ERR_INVALID_ARG, "bad sizes");
    const int G = Hq / Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
        return fail(PA_ERR_UNSUPPORTED, "group size %d (1, 2, 4, 8 or 16)", G);
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(PA_ERR_INVALID_ARG, "scale must be finite and positive");
    if (S == 0 || T == 0 || max_query_len == 0) return PA_OK;
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens ||
        !query_start)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!pa::aligned16(out) || !pa::aligned16(q) || !pa::aligned16(key_cache) ||
        !pa::aligned16(value_cache))
        return fail(PA_ERR_INVALID_ARG, "out, q and the caches must be 16-byte aligned");
    const int TQ = pf::kBM / G;
    const long long n_qt = ((long long)max_query_len + TQ - 1) / TQ;
    const long long n_pairs = (n_qt + 1) / 2;             // two query tiles per CTA
    if (S > 65535 || n_pairs > 65535 || Hkv > 65535)
        return fail(PA_ERR_UNSUPPORTED, "grid too large (S %d, query tiles %lld)", S, n_qt);
    if (NB > 0x7fffffffLL) return fail(PA_ERR_INVALID_ARG, "NB must fit int32 block ids");

    CUtensorMap mq, mk, mv;
    pa_status st = pa::make_rows_map(&mq, q, q_dt, T, Hq, D, G, TQ);
    if (st) return st;
    st = pa::make_cache_map(&mk, key_cache, cache_dt, NB, bs, Hkv, D);
    if (st) return st;
    st = pa::make_cache_map(&mv, value_cache, cache_dt, NB, bs, Hkv, D);
    if (st) return st;
    unsigned int* err = pa::device_error_word();
    if (!err) return PA_ERR_CUDA;

    pf::Params p = {};
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.err = err;
    p.NB = NB;
    p.S = S;
    p.Hq = Hq;
    p.G = G;
    p.log2G = __builtin_ctz((unsigned)G);
    p.TQ = TQ;
    p.MB = MB;
    p.bs = bs;
    p.log2bs = __builtin_ctz((unsigned)bs);
    p.max_qlen = max_query_len;
    p.n_pairs = (int)n_pairs;
    p.sl = scale * 1.4426950408889634f;
    p.pair_group = pf::kPairGroup;

    const dim3 grid((unsigned)(Hkv * pf::kPairGroup), (unsigned)S,
                    (unsigned)((n_pairs + pf::kPairGroup - 1) / pf::kPairGroup));
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (D == 128 && (pa::decode_select_mode() & 64)) {
        // the two query tiles of a pair on a pair of SMs (cta_group::2)
        const dim3 grid2(2 * grid.x, grid.y, grid.z);
        e = q_dt == PA_BF16 ? pf::launch2<PA_BF16>(mq, mk, mv, p, grid2, cs)
                            : pf::launch2<PA_F16>(mq, mk, mv, p, grid2, cs);
        if (e != cudaSuccess) return pa::cuda_fail(e, "prefill launch");
        return PA_OK;
    }
    if (q_dt == PA_BF16)
        e = D == 64 ? pf::launch<PA_BF16, 64>(mq, mk, mv, p, grid, cs)
                    : pf::launch<PA_BF16, 128>(mq, mk, mv, p, grid, cs);
    else
        e = D == 64 ? pf::launch<PA_F16, 64>(mq, mk, mv, p, grid, cs)
                    : pf::launch<PA_F16, 128>(mq, mk, mv, p, grid, cs);
    if (e != cudaSuccess) return pa::cuda_fail(e, "prefill launch");
    return PA_OK;
}
