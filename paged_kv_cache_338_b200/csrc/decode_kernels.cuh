// Paged decode attention kernels for sm_100a.
//
// What is computed ("PagedAttention 机制" §5.3.4; intelliparadigm PagedAttention
// article §2.3; "01. PagedAttention 详解" §4): for sequence s, query head h and
// kv head g = h / G, over the n_s tokens whose keys sit at
// key_cache[block_tables[s][i / bs], i % bs, g, :],
//     out = softmax(scale * K q) V.
//
// How (B200 design, not the pages' sketch):
//  * One CTA per (split-K partition, kv head [, head chunk], sequence).  It
//    streams the partition's physical blocks of ONE kv head through a ring of
//    STAGES shared-memory stages.  A stage holds the K tile and the V tile of
//    one block: bs rows of D elements each (bs * D * elt bytes, rows strided by
//    Hkv * D * elt in HBM).  Each tile arrives by one 5-D tensor-map (TMA)
//    load whose coordinates come from the block table, so the gather needs no
//    address arithmetic in the consumers; out-of-range ids read zeros.
//  * A producer warp (one elected lane) issues the loads; per-stage "full"
//    mbarriers carry the byte count, per-stage "empty" mbarriers return the
//    stage.  Every wait is bounded in time; on timeout the CTA records
//    PA_DEV_WAIT_TIMEOUT, drains its in-flight copies (again bounded) and
//    returns without writing.
//  * Consumer warp w takes blocks w, w + NW, ... and keeps its own online
//    softmax state (running max m, sum l, accumulator o) in the base-2
//    domain (scores pre-multiplied by log2(e)); the warps are merged once at
//    the end through shared memory.  All G query heads of the kv head share
//    each K/V tile, so K/V is read from HBM once per kv head.
//  * Two consumers:
//      - SIMT: 8 lanes per token row, each lane holding D/8 dims; dot
//        products on FP32 FMA units with a 3-step butterfly; any dtype.
//      - MMA (GQA, 16-bit K/V): the G query rows padded to 8 (or 16) form the
//        A operand of mma.sync m16n8k16 (bf16/f16 in, fp32 accumulate):
//        S = Q K^T with K^T fed by ldmatrix from the swizzled tile, then
//        O += P V with V fed by ldmatrix.trans; P stays in registers (its
//        accumulator layout is the A-operand layout of the second product).
//  * With more than one partition, (m, l, o) go to the fp32 workspace and
//    decode_merge combines them; otherwise the CTA writes out directly.
//  * Short partitions (decode_partition<C, true>): one CTA streams several
//    consecutive partitions of one (sequence, kv head) without draining its
//    ring, closes each with the warp merge through an smem area of its own
//    and writes that partition's record, so the split and its reduce are
//    those of one CTA per partition while the start-up and drain of a CTA
//    are paid once per group.
#pragma once

#include <type_traits>

#include "pa_device.cuh"

namespace pa {
namespace dec {

struct Params {
    void* out;                   // [S, Hq, D] q dtype
    const void* q;               // [S, Hq, D]
    const int32_t* block_tables; // [S, MB]
    const int32_t* context_lens; // [S]
    float2* ws_ml;               // [S, Hq, max_parts] (m, l)   (split-K only)
    float* ws_o;                 // [S, Hq, max_parts, D]       (split-K only)
    unsigned int* err;           // sticky device error word
    int S, Hq, Hkv, MB;
    int max_parts;               // partitions per sequence in the grid
    int part_blocks;             // blocks per partition (0: the whole sequence)
    int part_tokens;             // part_blocks * bs
    int max_ctx;                 // upper bound the grid / workspace were sized for
    int evict_first;             // 1: stream K/V with an L2 evict-first hint
    int heads_fastest;           // grid order: 1 = (kv head, partition, seq), 0 = (partition, kv head, seq)
    int bs;                      // block size (tokens)
    int balanced;                // 1: persistent work-balanced grid (decode_balanced)
    int2* ws_item;               // balanced: per item (first CTA, last CTA) holding its pieces
    int gc;                      // query heads per CTA item (G for the tensor-core consumer)
    int64_t ws_rows;             // balanced: partial rows the workspace holds
    int64_t NB;
    float qk_scale;              // scale * k_scale * log2(e)
    float v_scale;
    int prefix_parts;            // shared-prefix decode: leading partitions another kernel
                                 // wrote for sequences whose table starts with row 0's blocks
    int force_ws;                // 1: every sequence's partials go through the workspace
    int fuse_prefix_blocks;      // > 0: shared-prefix decode with one CTA per (sequence, kv
                                 // head) over the suffix past this many blocks; its epilogue
                                 // merges the prefix_parts prefix records and writes the output
    int part_group;              // plain split-K: consecutive partitions one CTA streams (>= 1),
                                 // still one record per partition
    int whole_items;             // balanced grid only: 1 = every item stays on one CTA (CTA
                                 // ranges end at item boundaries), whose output it writes;
                                 // with fuse_prefix_blocks the regular items read their suffix
                                 // and fold the prefix_parts prefix records in
    int rec_smem;                // one CTA per suffix: bytes of dynamic shared memory past the
                                 // barriers for its prefix records, fetched by a bulk copy while
                                 // the suffix streams (0: copied into the stages afterwards)
};

// Record a wait that gave up, with the site that gave up (bits 16-23).
__device__ __forceinline__ void wait_timeout(const Params& p, unsigned site) {
    dev::raise_error(p.err, PA_DEV_WAIT_TIMEOUT | (site << 16));
}

// Context length of sequence s, clamped to what the grid, the workspace and
// the table row can hold; anything out of range is reported, never followed.
__device__ __forceinline__ int checked_len(const Params& p, int s, int bs) {
    int n = p.context_lens[s];
    const int lim = min(p.max_ctx, p.MB * bs);
    if (n < 0 || n > lim) {
        dev::raise_error(p.err, PA_DEV_BAD_CONTEXT);
        n = n < 0 ? 0 : lim;
    }
    return n;
}

constexpr float kLog2e = 1.4426950408889634f;

// BS is the tokens of one stage; PB the tokens of one physical cache block.
// A stage holds PER = BS / PB consecutive blocks of a sequence (two blocks of
// 8 tokens make a 16-token stage, so an 8-token cache pays the per-stage
// costs -- barrier round trips, softmax updates, half-empty MMA tiles -- once
// per 16 tokens).
//
// HG is the kv heads one CTA serves.  With HG > 1 (= NW) every stage holds
// the rows of HG neighbouring kv heads, fetched by one tensor-map copy per
// block and 128-byte segment (the heads' rows of a token are adjacent in
// memory, so a copy reads HG x 128 contiguous bytes per token instead of 128),
// and consumer warp w serves kv head w of the group over every stage: no warp
// merge, no split of a head's blocks between warps.
template <int DT_, int QT_, int BS_, int D_, int GC_, bool MMA_, int MROWS_ = 8, int PB_ = BS_,
          int HG_ = 1>
struct Cfg {
    static constexpr int DT = DT_, QT = QT_, BS = BS_, D = D_, GC = GC_, MROWS = MROWS_;
    static constexpr int PB = PB_, PER = BS_ / PB_, HG = HG_;
    static constexpr bool MMA = MMA_;
    static constexpr int E = dev::Storage<DT>::bytes;
    static constexpr int R = D * E;          // bytes of one token row of one kv head
    static constexpr int CH = R / 128;       // 128-byte segments per row
    static constexpr int EPS = 128 / E;      // elements per segment
    static constexpr int EPC = 16 / E;       // elements per 16-byte chunk
    static constexpr int DPL = D / 8;        // dims per lane (SIMT consumer)
    static constexpr int TILE = HG * BS * R; // bytes of the K (or V) tiles of a stage
    static constexpr int STAGE = 2 * TILE;
    static constexpr int SEGSTRIDE = HG * BS * 128;   // bytes between 128-byte segments
    static constexpr int NW = 4;             // consumer warps
    static constexpr int THREADS = (NW + 1) * 32;
    static constexpr int BUDGET = 64 * 1024;                  // 3 CTAs per SM fit
    static constexpr int COMBINE_FLOATS = NW * GC * (D + 2);   // warp merge reuses the stages
    static constexpr int STAGES_RAW = BUDGET / STAGE;
    static constexpr int STAGES_MIN_C = (COMBINE_FLOATS * 4 + STAGE - 1) / STAGE;
    static constexpr int OWN = HG > 1 ? 1 : NW;  // stage count granule (see below)
    static constexpr int STAGES_MIN = STAGES_MIN_C > (HG > 1 ? 2 : NW) ? STAGES_MIN_C
                                                                       : (HG > 1 ? 2 : NW);
    static constexpr int STAGES_MAX = STAGES_MIN > 16 ? STAGES_MIN : 16;
    static constexpr int STAGES_CLAMPED = STAGES_RAW < STAGES_MIN ? STAGES_MIN
                                          : (STAGES_RAW > STAGES_MAX ? STAGES_MAX : STAGES_RAW);
    // One head per CTA: block j goes to consumer warp j % NW and to stage
    // j % STAGES.  With STAGES a multiple of NW every stage has exactly one
    // consumer warp, so a warp waiting on a stage's "full" barrier is never
    // more than one phase behind it and the parity wait cannot mistake an
    // older, still pending phase for the one it wants.  Round down, or up when
    // the warp merge needs the room.  Head groups: every warp consumes every
    // stage and the stage's "empty" barrier waits for all of them, so no warp
    // can fall a phase behind either.
    static constexpr int STAGES_DOWN = STAGES_CLAMPED / OWN * OWN;
    static constexpr int STAGES = STAGES_DOWN >= STAGES_MIN ? STAGES_DOWN
                                  : (STAGES_MIN + OWN - 1) / OWN * OWN;
    static constexpr size_t SMEM = 1024 /*align slack*/ + size_t(STAGES) * STAGE + 2 * 8 * STAGES;
    static_assert(R == 128 || R == 256 || R == 512, "row bytes must be 128, 256 or 512");
    static_assert(BS == 8 || BS == 16 || BS == 32, "block size");
    static_assert(PER == 1 || (PER == 2 && PB == 8), "a stage holds one block, or two of 8 tokens");
    static_assert(HG > 1 || STAGES % NW == 0, "each stage must have a single consumer warp");
    static_assert(HG == 1 || (HG == NW && MMA), "a head group is one kv head per consumer warp");
    static_assert(COMBINE_FLOATS * 4 <= STAGES * STAGE, "combine area must fit in the stages");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Tiles are stored segment-major: [128-byte segment][token][128 bytes], each
// 128-byte row swizzled by its token index (TMA SWIZZLE_128B, one box per
// segment).  Eight consecutive tokens of one 16-byte chunk column therefore
// sit in eight different bank groups, which keeps ldmatrix conflict-free.
// With head groups a segment is [block of the stage][head][token][128 bytes]
// and a head's tile starts at its own offset (head * PB * 128); with one head,
// [token][128 bytes].  A head's block slices are 1024-byte aligned, so a
// row's swizzle phase is its token index either way.
template <class C>
__device__ __forceinline__ int tile_row(int t) {
    return C::HG == 1 ? t : (t / C::PB) * C::HG * C::PB + (t % C::PB);
}
template <class C>
__device__ __forceinline__ uint32_t tile_off(int t, int seg, int chunk) {
    return (uint32_t)seg * C::SEGSTRIDE + dev::swz128(tile_row<C>(t), chunk);
}

// ------------------------------------------------------------------ producer
// One warp.  Block ids are fetched 32 at a time (one per lane) and handed out
// with shuffles, so the issue loop never waits on a dependent global load.
// Stages whose slot has not been used yet (the CTA's first ring) need no wait
// on an "empty" barrier: one lane each issues them, side by side; every later
// stage is issued by lane 0 once its slot is free.
//
// A lane's id of the first 32 blocks can be loaded ahead of time (while the
// CTA still reads its context length and sets up its barriers):
// table_entry_ahead() loads it for a guessed first physical block, and
// produce() uses it when the guess was right (pre_pblk0 == blk0 * PER).
__device__ __forceinline__ int table_entry_ahead(const Params& p, int s, int pblk0_guess) {
    const int i = pblk0_guess + (threadIdx.x & 31);
    return (pblk0_guess >= 0 && i < p.MB) ? __ldg(p.block_tables + (size_t)s * p.MB + i) : 0;
}

// Issue stage slot `st`: `have` (>= 1) physical blocks id[0 .. have-1] of
// kv head kvh (the first head of the group), every 128-byte segment of K and
// V, completing on the slot's "full" barrier.
template <class C>
__device__ __forceinline__ void issue_stage(const CUtensorMap* tmk, const CUtensorMap* tmv,
                                            const Params& p, const int (&id)[C::PER], int have,
                                            int kvh, int st, uint8_t* stages, uint32_t full0,
                                            uint64_t pol) {
    const uint32_t bar = full0 + 8 * st;
    const uint32_t dk = dev::smem_addr(stages + (size_t)st * C::STAGE);
    dev::mbar_arrive_expect_tx(bar, (uint32_t)have * 2 * C::HG * C::PB * C::R);
    #pragma unroll
    for (int r = 0; r < C::PER; ++r) {
        if (r >= have) break;
        if (id[r] < 0 || (int64_t)id[r] >= p.NB) dev::raise_error(p.err, PA_DEV_BAD_BLOCK);
        #pragma unroll
        for (int c = 0; c < C::CH; ++c) {
            const uint32_t off = c * C::SEGSTRIDE + r * C::HG * C::PB * 128;
            if constexpr (C::HG == 1) {   // map {D, Hkv, bs, NB}
                dev::tma_load_4d(dk + off, tmk, bar, c * C::EPS, kvh, 0, id[r], pol);
                dev::tma_load_4d(dk + C::TILE + off, tmv, bar, c * C::EPS, kvh, 0, id[r], pol);
            } else {                      // map {D, bs, Hkv, NB}, kvh the first head
                dev::tma_load_4d(dk + off, tmk, bar, c * C::EPS, 0, kvh, id[r], pol);
                dev::tma_load_4d(dk + C::TILE + off, tmv, bar, c * C::EPS, 0, kvh, id[r], pol);
            }
        }
    }
}

template <class C>
__device__ __forceinline__ void produce(const CUtensorMap* tmk, const CUtensorMap* tmv,
                                        const Params& p, const int32_t* bt_row, int blk0, int nblk,
                                        int nphys, int kvh, uint8_t* stages, uint32_t full0,
                                        uint32_t empty0, volatile int* s_abort, int* k_io,
                                        int pre_pblk0 = -1, int pre = 0) {
    // Streams stages [blk0, blk0 + nblk) of one (sequence, kv head) through the
    // stage ring; *k_io is the CTA's running stage counter (slot = k % STAGES).
    // Stage j holds physical blocks (blk0 + j) * PER + r, r < PER, of which the
    // first nphys (counted from blk0 * PER) exist; a stage past them is left
    // part-filled (its tokens are past the sequence's length).
    const int lane = threadIdx.x & 31;
    const uint64_t pol = p.evict_first ? dev::policy_evict_first() : dev::policy_evict_normal();
    const int pblk0 = blk0 * C::PER;
    int k = *k_io;
    for (int jb = 0; jb < nblk * C::PER; jb += 32) {          // 32 physical ids per round
        const int mine = jb + lane >= nphys ? 0
                         : (jb == 0 && pre_pblk0 == pblk0) ? pre
                                                           : __ldg(bt_row + pblk0 + jb + lane);
        const int cnt = min(32, nblk * C::PER - jb) / C::PER;   // stages of this round
        // the round's stages in never-used slots: lane jj issues stage jj
        const int nfree = max(0, min(cnt, C::STAGES - k));
        {
            int id[C::PER];
            #pragma unroll
            for (int r = 0; r < C::PER; ++r)
                id[r] = __shfl_sync(0xffffffffu, mine, (lane * C::PER + r) & 31);
            if (lane < nfree)
                issue_stage<C>(tmk, tmv, p, id, min(C::PER, nphys - (jb + lane * C::PER)), kvh,
                               (k + lane) % C::STAGES, stages, full0, pol);
        }
        k += nfree;
        for (int jj = nfree; jj < cnt; ++jj) {
            int id[C::PER];
            #pragma unroll
            for (int r = 0; r < C::PER; ++r) id[r] = __shfl_sync(0xffffffffu, mine, jj * C::PER + r);
            int stop = 0;
            if (lane == 0) {
                const int st = k % C::STAGES;
                const uint32_t par = ((k / C::STAGES) & 1) ^ 1;
                if (!dev::mbar_wait_bounded(empty0 + 8 * st, par)) {
                    wait_timeout(p, 1);
                    *s_abort = 1;
                    stop = 1;
                } else {
                    issue_stage<C>(tmk, tmv, p, id, min(C::PER, nphys - (jb + jj * C::PER)), kvh,
                                   st, stages, full0, pol);
                }
            }
            stop = __shfl_sync(0xffffffffu, stop, 0);
            if (stop) {
                *k_io = k;
                return;
            }
            ++k;
        }
    }
    *k_io = k;
}

// --------------------------------------------------------- SIMT consumer
template <class C>
struct SimtState {
    float q[C::GC][C::DPL];
    float acc[C::GC][C::DPL];
    float m[C::GC];
    float l[C::GC];
};

template <class C>
__device__ __forceinline__ void simt_load_q(SimtState<C>& st, const Params& p, int s, int h0) {
    const int lane = threadIdx.x & 31;
    const int l8 = lane & 7;
    #pragma unroll
    for (int g = 0; g < C::GC; ++g) {
        const size_t base = ((size_t)s * p.Hq + h0 + g) * C::D;
        #pragma unroll
        for (int k = 0; k < C::CH; ++k)
            #pragma unroll
            for (int e = 0; e < C::EPC; ++e)
                st.q[g][k * C::EPC + e] =
                    dev::load_q<C::QT>(p.q, base + k * C::EPS + l8 * C::EPC + e) * p.qk_scale;
        #pragma unroll
        for (int j = 0; j < C::DPL; ++j) st.acc[g][j] = 0.f;
        st.m[g] = -INFINITY;
        st.l[g] = 0.f;
    }
}

template <class C>
__device__ __forceinline__ void simt_reset(SimtState<C>& st) {
    #pragma unroll
    for (int g = 0; g < C::GC; ++g) {
        #pragma unroll
        for (int j = 0; j < C::DPL; ++j) st.acc[g][j] = 0.f;
        st.m[g] = -INFINITY;
        st.l[g] = 0.f;
    }
}

// Dims of token row t of a tile held by this lane, as floats.
template <class C>
__device__ __forceinline__ void simt_row(const uint8_t* tile, int t, int l8, float* f) {
    #pragma unroll
    for (int k = 0; k < C::CH; ++k) {
        const uint4 r = *reinterpret_cast<const uint4*>(tile + tile_off<C>(t, k, l8));
        dev::Chunk<C::DT>::to_float(r, f + k * C::EPC);
    }
}

template <class C>
__device__ __forceinline__ void simt_block(SimtState<C>& st, const uint8_t* ktile,
                                           const uint8_t* vtile, int nvalid) {
    const int lane = threadIdx.x & 31;
    const int l8 = lane & 7, grp = lane >> 3;
    constexpr int SUB = C::BS < 16 ? C::BS : 16;   // tokens per online-softmax update
    constexpr int IT = SUB / 4;                     // 4 tokens per warp pass
    float f[C::DPL];
    #pragma unroll
    for (int sb = 0; sb < C::BS / SUB; ++sb) {
        float sc[IT][C::GC];
        #pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int t = sb * SUB + it * 4 + grp;
            simt_row<C>(ktile, t, l8, f);
            #pragma unroll
            for (int g = 0; g < C::GC; ++g) {
                float a = 0.f;
                #pragma unroll
                for (int j = 0; j < C::DPL; ++j) a = fmaf(st.q[g][j], f[j], a);
                a += __shfl_xor_sync(0xffffffffu, a, 1);
                a += __shfl_xor_sync(0xffffffffu, a, 2);
                a += __shfl_xor_sync(0xffffffffu, a, 4);
                sc[it][g] = (t < nvalid) ? a : -INFINITY;
            }
        }
        #pragma unroll
        for (int g = 0; g < C::GC; ++g) {
            float bm = sc[0][g];
            #pragma unroll
            for (int it = 1; it < IT; ++it) bm = fmaxf(bm, sc[it][g]);
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
            if (bm > st.m[g]) {                       // warp-uniform
                const float alpha = exp2f(st.m[g] - bm);
                st.l[g] *= alpha;
                #pragma unroll
                for (int j = 0; j < C::DPL; ++j) st.acc[g][j] *= alpha;
                st.m[g] = bm;
            }
        }
        #pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int t = sb * SUB + it * 4 + grp;
            if (t < nvalid) {
                simt_row<C>(vtile, t, l8, f);
                #pragma unroll
                for (int g = 0; g < C::GC; ++g) {
                    const float pr = exp2f(sc[it][g] - st.m[g]);
                    st.l[g] += pr;
                    #pragma unroll
                    for (int j = 0; j < C::DPL; ++j) st.acc[g][j] = fmaf(pr, f[j], st.acc[g][j]);
                }
            }
        }
    }
}

// Reduce the four token groups of the warp and publish (m, l, acc) to smem.
template <class C>
__device__ __forceinline__ void simt_publish(SimtState<C>& st, float* cm, float* cl, float* co,
                                             int w, int gs = C::GC) {
    const int lane = threadIdx.x & 31;
    const int l8 = lane & 7, grp = lane >> 3;
    #pragma unroll
    for (int g = 0; g < C::GC; ++g) {
        float l = st.l[g];
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        #pragma unroll
        for (int j = 0; j < C::DPL; ++j) {
            float a = st.acc[g][j];
            a += __shfl_xor_sync(0xffffffffu, a, 8);
            a += __shfl_xor_sync(0xffffffffu, a, 16);
            st.acc[g][j] = a;
        }
        if (lane == 0) {
            cm[w * gs + g] = st.m[g];
            cl[w * gs + g] = l;
        }
        if (grp == 0) {
            #pragma unroll
            for (int k = 0; k < C::CH; ++k)
                #pragma unroll
                for (int e = 0; e < C::EPC; ++e)
                    co[(w * gs + g) * C::D + k * C::EPS + l8 * C::EPC + e] =
                        st.acc[g][k * C::EPC + e];
        }
    }
}

// ---------------------------------------------------------- MMA consumer
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

template <int DT>
__device__ __forceinline__ void mma16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    if constexpr (DT == PA_BF16) {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    } else {
        asm(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
}

template <int DT>
__device__ __forceinline__ void mma1688(float* c, uint32_t a0, uint32_t a1, uint32_t b0) {
    if constexpr (DT == PA_BF16) {
        asm(
            "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(b0));
    } else {
        asm(
            "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
            "{%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a0), "r"(a1), "r"(b0));
    }
}

// Round two floats into a packed 16-bit pair (lower index in the low half),
// and return the rounded values.
template <int DT>
__device__ __forceinline__ uint32_t pack2(float x, float y, float& rx, float& ry) {
    if constexpr (DT == PA_BF16) {
        __nv_bfloat162 v = __floats2bfloat162_rn(x, y);
        float2 r = __bfloat1622float2(v);
        rx = r.x; ry = r.y;
        return *reinterpret_cast<uint32_t*>(&v);
    } else {
        __half2 v = __floats2half2_rn(x, y);
        float2 r = __half22float2(v);
        rx = r.x; ry = r.y;
        return *reinterpret_cast<uint32_t*>(&v);
    }
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// Tensor-core consumer.  Per KV block of bs tokens and the query heads of one
// kv head (NH tiles of 8 heads):
//   S^T [tokens x heads] = K [tokens x D] . Q^T [D x heads]    (m16n8k16, tokens on M)
//   P^T = 2^(S^T - m), rounded to 16 bits; movmatrix turns its accumulator
//         fragments into the B fragments of the second product
//   O^T [D x heads]     += V^T [D x tokens] . P^T [tokens x heads]
// A thread owns heads 2*tig, 2*tig+1 of each head tile for softmax state.
// 16-bit caches feed both products straight from the stage with ldmatrix.
// An fp8 cache computes in f16: K fragments come from ldmatrix on the bytes
// (a b16 lane holds 2 codes, so a thread receives 4 consecutive dims) and are
// widened with cvt.f16x2.e4m3x2; the contraction index is permuted the same
// way on Q, so logical k (2t, 2t+1 | 2t+8, 2t+9) of a 16-dim step is physical
// dim (4t, 4t+1 | 4t+2, 4t+3).  V^T fragments also come straight from the
// codes: ldmatrix.trans on 16-bit units hands a thread tokens (2t, 2t+1) of
// dims (2g, 2g+1), a byte permute pairs the two tokens of one dim and the
// pair is widened; so logical row g of an O^T m-tile is physical dim 2g and
// row g + 8 is dim 2g + 1 (undone when the accumulators are published).
// Codes of tokens past the valid ones are cleared before widening (a zero
// weight times a NaN code would still be NaN).
template <class C>
struct MmaState {
    static constexpr bool FP8 = C::DT == PA_FP8_E4M3;
    static constexpr int CT = FP8 ? PA_F16 : C::DT;   // tensor-core input type
    static constexpr int NH = C::MROWS / 8;  // head tiles of 8
    static constexpr int KS = C::D / 16;     // k-steps over D
    static constexpr int MD = C::D / 16;     // m-tiles of O^T
    uint32_t qb[NH][KS][2];                  // B fragments of Q^T
    float o[NH][MD][4];                      // O^T accumulators
    float m[NH][2], l[NH][2];                // heads 2*tig, 2*tig+1 of each tile
};

template <int QT>
__device__ __forceinline__ uint32_t to_f16x2(uint32_t w) {
    if constexpr (QT == PA_F16) {
        return w;
    } else {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
        __half2 h = __floats2half2_rn(f.x, f.y);
        return *reinterpret_cast<uint32_t*>(&h);
    }
}

// Four E4M3 codes (bytes 0..3 of w) to two f16x2 words: lo = (code 0, code 1),
// hi = (code 2, code 3).  Every E4M3 value is an f16 value, so the conversion
// is exact; the word is split into its 16-bit halves inside the asm so that
// each half feeds its conversion directly.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

template <class C>
__device__ __forceinline__ void mma_load_q(MmaState<C>& st, const Params& p, int s, int h0,
                                           int G) {
    using S = MmaState<C>;
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    const uint32_t* q32 = static_cast<const uint32_t*>(p.q);
    #pragma unroll
    for (int nh = 0; nh < S::NH; ++nh) {
        const int head = nh * 8 + gid;
        const size_t base = (((size_t)s * p.Hq + h0 + head) * C::D) / 2;
        #pragma unroll
        for (int ks = 0; ks < S::KS; ++ks) {
            uint32_t b0 = 0u, b1 = 0u;
            if (head < G) {
                if constexpr (S::FP8) {
                    // physical dims ks*16 + 4tig, +1  and  ks*16 + 4tig + 2, +3
                    b0 = to_f16x2<C::QT>(__ldg(q32 + base + ks * 8 + 2 * tig));
                    b1 = to_f16x2<C::QT>(__ldg(q32 + base + ks * 8 + 2 * tig + 1));
                } else {
                    // dims ks*16 + 2tig, +1  and  ks*16 + 8 + 2tig, +1
                    b0 = __ldg(q32 + base + ks * 8 + tig);
                    b1 = __ldg(q32 + base + ks * 8 + 4 + tig);
                }
            }
            st.qb[nh][ks][0] = b0;
            st.qb[nh][ks][1] = b1;
        }
        #pragma unroll
        for (int md = 0; md < S::MD; ++md)
            #pragma unroll
            for (int i = 0; i < 4; ++i) st.o[nh][md][i] = 0.f;
        st.m[nh][0] = st.m[nh][1] = -INFINITY;
        st.l[nh][0] = st.l[nh][1] = 0.f;
    }
}

// smem address of 16-byte chunk c (over the whole row) of token row t
template <class C>
__device__ __forceinline__ uint32_t chunk_addr(uint32_t tile, int t, int c) {
    return tile + tile_off<C>(t, c >> 3, c & 7);
}

template <class C>
__device__ __forceinline__ void mma_block(MmaState<C>& st, uint8_t* ktile_p, uint8_t* vtile_p,
                                          int nvalid, float qk_scale) {
    using S = MmaState<C>;
    constexpr int BS = C::BS;
    constexpr int CT = S::CT;
    constexpr int MT = BS >= 16 ? BS / 16 : 1;   // token m-tiles of S^T
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2;
    const uint32_t ktile = dev::smem_addr(ktile_p);

    // ---- S^T = K Q^T --------------------------------------------------------
    float sc[MT][S::NH][4];
    #pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        #pragma unroll
        for (int nh = 0; nh < S::NH; ++nh)
            #pragma unroll
            for (int i = 0; i < 4; ++i) sc[mt][nh][i] = 0.f;
        if constexpr (S::FP8) {
            // a 16-byte chunk is one 16-dim k-step; ldmatrix rows are 8 tokens
            float sc8_odd[S::NH][4];
            #pragma unroll
            for (int nh = 0; nh < S::NH; ++nh)
                #pragma unroll
                for (int i = 0; i < 4; ++i) sc8_odd[nh][i] = 0.f;
            #pragma unroll
            for (int ks = 0; ks < S::KS; ks += 2) {
                uint32_t r0, r1, r2, r3;
                if constexpr (BS >= 16) {
                    // (tok 0-7, chunk ks) (tok 8-15, ks) (tok 0-7, ks+1) (tok 8-15, ks+1)
                    ldsm_x4(chunk_addr<C>(ktile, mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7),
                                          ks + (lane >> 4)),
                            r0, r1, r2, r3);
                } else {
                    // (tok 0-7, chunk ks) (tok 0-7, ks+1); rows 8-15 of A are zero
                    uint32_t u0, u1;
                    ldsm_x4(chunk_addr<C>(ktile, lane & 7, ks + ((lane >> 3) & 1)), r0, r2, u0, u1);
                    r1 = r3 = 0u;
                }
                uint32_t a00, a02, a10, a12, a01 = 0u, a03 = 0u, a11 = 0u, a13 = 0u;
                e4m3x4_to_f16x2(r0, a00, a02);
                e4m3x4_to_f16x2(r2, a10, a12);
                if constexpr (BS >= 16) {
                    e4m3x4_to_f16x2(r1, a01, a03);
                    e4m3x4_to_f16x2(r3, a11, a13);
                }
                #pragma unroll
                for (int nh = 0; nh < S::NH; ++nh) {
                    mma16816<CT>(sc[mt][nh], a00, a01, a02, a03, st.qb[nh][ks][0], st.qb[nh][ks][1]);
                    mma16816<CT>(sc8_odd[nh], a10, a11, a12, a13, st.qb[nh][ks + 1][0],
                                 st.qb[nh][ks + 1][1]);
                }
            }
            #pragma unroll
            for (int nh = 0; nh < S::NH; ++nh)
                #pragma unroll
                for (int i = 0; i < 4; ++i) sc[mt][nh][i] += sc8_odd[nh][i];
        } else if constexpr (BS >= 16) {
            // two independent accumulation chains (even / odd k-steps) halve
            // the dependent mma latency of the product
            float sc_odd[S::NH][4];
            #pragma unroll
            for (int nh = 0; nh < S::NH; ++nh)
                #pragma unroll
                for (int i = 0; i < 4; ++i) sc_odd[nh][i] = 0.f;
            #pragma unroll
            for (int ks = 0; ks < S::KS; ++ks) {
                // matrices: (tok 0-7, chunk 2ks) (tok 8-15, 2ks) (tok 0-7, 2ks+1) (tok 8-15, 2ks+1)
                uint32_t a0, a1, a2, a3;
                ldsm_x4(chunk_addr<C>(ktile, mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7),
                                      2 * ks + (lane >> 4)),
                        a0, a1, a2, a3);
                #pragma unroll
                for (int nh = 0; nh < S::NH; ++nh)
                    mma16816<CT>((ks & 1) ? sc_odd[nh] : sc[mt][nh], a0, a1, a2, a3,
                                 st.qb[nh][ks][0], st.qb[nh][ks][1]);
            }
            #pragma unroll
            for (int nh = 0; nh < S::NH; ++nh)
                #pragma unroll
                for (int i = 0; i < 4; ++i) sc[mt][nh][i] += sc_odd[nh][i];
        } else {
            // 8 tokens: rows 8-15 of the A operand are zero
            #pragma unroll
            for (int ks = 0; ks < S::KS; ks += 2) {
                uint32_t a0, a2, b0, b2;   // chunks 2ks, 2ks+1, 2ks+2, 2ks+3 of tokens 0-7
                ldsm_x4(chunk_addr<C>(ktile, lane & 7, 2 * ks + (lane >> 3)), a0, a2, b0, b2);
                #pragma unroll
                for (int nh = 0; nh < S::NH; ++nh) {
                    mma16816<CT>(sc[mt][nh], a0, 0u, a2, 0u, st.qb[nh][ks][0], st.qb[nh][ks][1]);
                    mma16816<CT>(sc[mt][nh], b0, 0u, b2, 0u, st.qb[nh][ks + 1][0],
                                 st.qb[nh][ks + 1][1]);
                }
            }
        }
    }
    // ---- online softmax over the block's tokens, per head ------------------
    #pragma unroll
    for (int nh = 0; nh < S::NH; ++nh) {
        float bm0 = -INFINITY, bm1 = -INFINITY;
        #pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int t0 = mt * 16 + gid, t1 = t0 + 8;
            const bool v0 = t0 < nvalid, v1 = (BS >= 16) && t1 < nvalid;
            sc[mt][nh][0] = v0 ? sc[mt][nh][0] * qk_scale : -INFINITY;
            sc[mt][nh][1] = v0 ? sc[mt][nh][1] * qk_scale : -INFINITY;
            sc[mt][nh][2] = v1 ? sc[mt][nh][2] * qk_scale : -INFINITY;
            sc[mt][nh][3] = v1 ? sc[mt][nh][3] * qk_scale : -INFINITY;
            bm0 = fmaxf(bm0, fmaxf(sc[mt][nh][0], sc[mt][nh][2]));
            bm1 = fmaxf(bm1, fmaxf(sc[mt][nh][1], sc[mt][nh][3]));
        }
        #pragma unroll
        for (int x = 4; x <= 16; x <<= 1) {
            bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, x));
            bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, x));
        }
        const bool grow = bm0 > st.m[nh][0] || bm1 > st.m[nh][1];
        if (__any_sync(0xffffffffu, grow)) {
            const float m0 = fmaxf(st.m[nh][0], bm0), m1 = fmaxf(st.m[nh][1], bm1);
            const float al0 = exp2f(st.m[nh][0] - m0), al1 = exp2f(st.m[nh][1] - m1);  // 0 from -inf
            st.m[nh][0] = m0;
            st.m[nh][1] = m1;
            st.l[nh][0] *= al0;
            st.l[nh][1] *= al1;
            #pragma unroll
            for (int md = 0; md < S::MD; ++md) {
                st.o[nh][md][0] *= al0; st.o[nh][md][2] *= al0;
                st.o[nh][md][1] *= al1; st.o[nh][md][3] *= al1;
            }
        }
    }
    // P^T fragments -> B fragments of O^T += V^T P^T (via an in-register transpose)
    uint32_t pb[MT][S::NH][2];
    #pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        #pragma unroll
        for (int nh = 0; nh < S::NH; ++nh) {
            float r0, r1, r2, r3;
            const uint32_t x = pack2<CT>(exp2f(sc[mt][nh][0] - st.m[nh][0]),
                                         exp2f(sc[mt][nh][1] - st.m[nh][1]), r0, r1);
            st.l[nh][0] += r0;
            st.l[nh][1] += r1;
            pb[mt][nh][0] = movmatrix_t(x);                 // tokens mt*16 + 0..7
            if constexpr (BS >= 16) {
                const uint32_t y = pack2<CT>(exp2f(sc[mt][nh][2] - st.m[nh][0]),
                                             exp2f(sc[mt][nh][3] - st.m[nh][1]), r2, r3);
                st.l[nh][0] += r2;
                st.l[nh][1] += r3;
                pb[mt][nh][1] = movmatrix_t(y);             // tokens mt*16 + 8..15
            }
        }
    }
    // ---- O^T += V^T P^T ---------------------------------------------------------
    if constexpr (S::FP8) {
        const uint32_t vt = dev::smem_addr(vtile_p);
        const int tig = lane & 3;
        const bool tail = nvalid < BS;
        if constexpr (BS >= 16) {
            // one pass over the tile; TAIL: codes of tokens at or past nvalid are
            // zeroed first (a zero weight times a NaN code would still be NaN)
            auto pass = [&](auto tail_tag) {
                constexpr bool TAIL = decltype(tail_tag)::value;
                #pragma unroll
                for (int kt = 0; kt < MT; ++kt) {
                    // bytes 0-1 of a fragment word: token 2tig; bytes 2-3: token 2tig + 1
                    uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
                    if constexpr (TAIL) {
                        const int t0 = kt * 16 + 2 * tig;
                        keep0 = (t0 < nvalid ? 0x0000ffffu : 0u) | (t0 + 1 < nvalid ? 0xffff0000u : 0u);
                        keep1 = (t0 + 8 < nvalid ? 0x0000ffffu : 0u) | (t0 + 9 < nvalid ? 0xffff0000u : 0u);
                    }
                    #pragma unroll
                    for (int md = 0; md < S::MD; md += 2) {
                        // matrices: (tok 0-7, chunk md) (tok 8-15, md) (tok 0-7, md+1) (tok 8-15, md+1)
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4_t(chunk_addr<C>(vt, kt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7),
                                                md + (lane >> 4)),
                                  r0, r1, r2, r3);
                        if constexpr (TAIL) {
                            r0 &= keep0;
                            r1 &= keep1;
                            r2 &= keep0;
                            r3 &= keep1;
                        }
                        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                        e4m3x4_to_f16x2(__byte_perm(r0, 0, 0x3120), a0, a1);
                        e4m3x4_to_f16x2(__byte_perm(r1, 0, 0x3120), a2, a3);
                        e4m3x4_to_f16x2(__byte_perm(r2, 0, 0x3120), b0, b1);
                        e4m3x4_to_f16x2(__byte_perm(r3, 0, 0x3120), b2, b3);
                        #pragma unroll
                        for (int nh = 0; nh < S::NH; ++nh) {
                            mma16816<CT>(st.o[nh][md], a0, a1, a2, a3, pb[kt][nh][0], pb[kt][nh][1]);
                            mma16816<CT>(st.o[nh][md + 1], b0, b1, b2, b3, pb[kt][nh][0],
                                         pb[kt][nh][1]);
                        }
                    }
                }
            };
            if (tail) pass(std::true_type{});
            else pass(std::false_type{});
        } else {
            uint32_t keep = 0xffffffffu;
            if (tail)
                keep = (2 * tig < nvalid ? 0x0000ffffu : 0u) | (2 * tig + 1 < nvalid ? 0xffff0000u : 0u);
            #pragma unroll
            for (int md = 0; md < S::MD; md += 4) {
                // matrices: tokens 0-7 of chunks md, md+1, md+2, md+3
                uint32_t r[4];
                ldsm_x4_t(chunk_addr<C>(vt, lane & 7, md + (lane >> 3)), r[0], r[1], r[2], r[3]);
                #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t a0, a1;
                    e4m3x4_to_f16x2(__byte_perm(r[i] & keep, 0, 0x3120), a0, a1);
                    #pragma unroll
                    for (int nh = 0; nh < S::NH; ++nh) mma1688<CT>(st.o[nh][md + i], a0, a1, pb[0][nh][0]);
                }
            }
        }
    } else {
        // the 16-bit tile itself, tail rows zeroed
        if (nvalid < BS) {
            // whole 128-byte rows of this warp's head, so the swizzle does not matter
            for (int i = lane; i < (BS - nvalid) * C::CH * 8; i += 32) {
                const int t = nvalid + i / (C::CH * 8), k = (i / 8) % C::CH;
                *reinterpret_cast<uint4*>(vtile_p + k * C::SEGSTRIDE + tile_row<C>(t) * 128 +
                                          (i % 8) * 16) = make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
        }
        const uint32_t vtile = dev::smem_addr(vtile_p);
        if constexpr (BS >= 16) {
            #pragma unroll
            for (int kt = 0; kt < MT; ++kt) {
                #pragma unroll
                for (int md = 0; md < S::MD; ++md) {
                    // matrices: (tok 0-7, chunk 2md) (tok 0-7, 2md+1) (tok 8-15, 2md) (tok 8-15, 2md+1)
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(chunk_addr<C>(vtile, kt * 16 + (lane >> 4) * 8 + (lane & 7),
                                            2 * md + ((lane >> 3) & 1)),
                              a0, a1, a2, a3);
                    #pragma unroll
                    for (int nh = 0; nh < S::NH; ++nh)
                        mma16816<CT>(st.o[nh][md], a0, a1, a2, a3, pb[kt][nh][0], pb[kt][nh][1]);
                }
            }
        } else {
            #pragma unroll
            for (int md = 0; md < S::MD; md += 2) {
                // matrices: tokens 0-7 of chunks 2md, 2md+1, 2md+2, 2md+3
                uint32_t a0, a1, b0, b1;
                ldsm_x4_t(chunk_addr<C>(vtile, lane & 7, 2 * md + (lane >> 3)), a0, a1, b0, b1);
                #pragma unroll
                for (int nh = 0; nh < S::NH; ++nh) {
                    mma1688<CT>(st.o[nh][md], a0, a1, pb[0][nh][0]);
                    mma1688<CT>(st.o[nh][md + 1], b0, b1, pb[0][nh][0]);
                }
            }
        }
    }
    if constexpr (!S::FP8) {
        if (nvalid < BS) dev::fence_proxy_async_smem();   // generic writes before the next TMA fill
    }
}

template <class C>
__device__ __forceinline__ void mma_publish(MmaState<C>& st, float* cm, float* cl, float* co,
                                            int w, int G, int gs = C::GC) {
    using S = MmaState<C>;
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2, tig = lane & 3;
    #pragma unroll
    for (int nh = 0; nh < S::NH; ++nh) {
        #pragma unroll
        for (int j = 0; j < 2; ++j) {
            float l = st.l[nh][j];
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            const int head = nh * 8 + 2 * tig + j;
            if (head < G) {
                if (gid == 0) {
                    cm[w * gs + head] = st.m[nh][j];
                    cl[w * gs + head] = l;
                }
                #pragma unroll
                for (int md = 0; md < S::MD; ++md) {
                    // fp8: logical rows gid, gid + 8 are dims 2 gid, 2 gid + 1
                    const int d0 = S::FP8 ? md * 16 + 2 * gid : md * 16 + gid;
                    const int d1 = S::FP8 ? d0 + 1 : d0 + 8;
                    co[(w * gs + head) * C::D + d0] = st.o[nh][md][j];
                    co[(w * gs + head) * C::D + d1] = st.o[nh][md][2 + j];
                }
            }
        }
    }
}

template <class C>
__device__ __forceinline__ void mma_reset(MmaState<C>& st) {
    using S = MmaState<C>;
    #pragma unroll
    for (int nh = 0; nh < S::NH; ++nh) {
        #pragma unroll
        for (int md = 0; md < S::MD; ++md)
            #pragma unroll
            for (int i = 0; i < 4; ++i) st.o[nh][md][i] = 0.f;
        st.m[nh][0] = st.m[nh][1] = -INFINITY;
        st.l[nh][0] = st.l[nh][1] = 0.f;
    }
}

// Barrier 1 over the consumer warps only (the producer keeps streaming).
template <class C>
__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(C::NW * 32) : "memory");
}
// The same barrier, returning whether any consumer thread passed `pred`.
template <class C>
__device__ __forceinline__ bool consumers_sync_or(bool pred) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)pred), "n"(C::NW * 32) : "memory");
    return r != 0;
}

// A whole item's outputs: the consumer warps' states (cm, cl, co in shared
// memory, stride gc) merged, then the prefix kernel's records of the item's
// heads folded in one after another (the split-K identity), four outputs per
// thread at a time with the loads of all their records in flight together
// (one round trip to L2 per four records instead of one per output).
template <class C>
__device__ __forceinline__ void fold_item(const Params& p, int s, int h0, int gc, const float* cm,
                                          const float* cl, const float* co) {
    constexpr int T = C::NW * 32, U = 4;
    const int total = gc * C::D;
    for (int base = threadIdx.x; base < total; base += U * T) {
        float M[U], L[U], O[U];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int idx = base + u * T;
            M[u] = -INFINITY;
            L[u] = 0.f;
            O[u] = 0.f;
            if (idx < total) {
                const int g = idx / C::D, dd = idx % C::D;
                float m = -INFINITY;
                #pragma unroll
                for (int w = 0; w < C::NW; ++w) m = fmaxf(m, cm[w * gc + g]);
                float l = 0.f, o = 0.f;
                if (m != -INFINITY) {
                    #pragma unroll
                    for (int w = 0; w < C::NW; ++w) {
                        const float f = exp2f(cm[w * gc + g] - m);
                        l = fmaf(f, cl[w * gc + g], l);
                        o = fmaf(f, co[(w * gc + g) * C::D + dd], o);
                    }
                }
                M[u] = m;
                L[u] = l;
                O[u] = o * p.v_scale;
            }
        }
        for (int pp0 = 0; pp0 < p.prefix_parts; pp0 += U) {
            float2 ml[U][U];
            float ro[U][U];
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                const int idx = base + u * T;
                const int g = idx / C::D, dd = idx % C::D;
                #pragma unroll
                for (int i = 0; i < U; ++i) {
                    if (idx < total && pp0 + i < p.prefix_parts) {
                        const size_t row = ((size_t)s * p.Hq + h0 + g) * p.max_parts + pp0 + i;
                        ml[u][i] = p.ws_ml[row];
                        ro[u][i] = p.ws_o[row * C::D + dd];
                    } else {
                        ml[u][i] = make_float2(-INFINITY, 0.f);
                        ro[u][i] = 0.f;
                    }
                }
            }
            #pragma unroll
            for (int u = 0; u < U; ++u) {
                #pragma unroll
                for (int i = 0; i < U; ++i) {
                    const float Mn = fmaxf(M[u], ml[u][i].x);
                    if (Mn == -INFINITY) continue;
                    const float a = exp2f(M[u] - Mn), b = exp2f(ml[u][i].x - Mn);
                    L[u] = L[u] * a + ml[u][i].y * b;
                    O[u] = O[u] * a + ro[u][i] * b;
                    M[u] = Mn;
                }
            }
        }
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int idx = base + u * T;
            if (idx < total)
                dev::store_out<C::QT>(p.out,
                                      ((size_t)s * p.Hq + h0 + idx / C::D) * C::D + idx % C::D,
                                      L[u] == 0.f ? 0.f : O[u] / L[u]);
        }
    }
}

// Smem bytes of the per-partition warp merge area of the grouped-partition
// mode (it cannot reuse the stages, which keep streaming).
template <class C>
constexpr size_t group_merge_bytes(int heads) {
    return size_t(C::NW) * heads * (C::D + 2) * sizeof(float);
}

// ----------------------------------------------------------------- kernel
// GROUPED: the grouped-partition instantiation (p.part_group > 1, plain
// split-K only); the other one is launched with p.part_group == 1.
template <class C, bool GROUPED>
__global__ void __launch_bounds__(C::THREADS, C::MMA ? 3 : 2)
decode_partition(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                 const Params p) {
    // Launched as a dependent of the kernel before it.  The shared-prefix
    // suffix pass reads nothing that kernel (the prefix kernel) writes until it
    // folds the prefix records in, so it waits there and streams its suffix
    // meanwhile; everything the kernels before that one wrote is complete when
    // this grid starts (the prefix kernel lets its dependents launch only after
    // its wait for the kernel before it returns, and every kernel of the step
    // waits for its predecessor before it finishes).
    if (threadIdx.x == C::NW * 32) {            // the producer's copies need both maps first
        dev::prefetch_tensormap(&tmk);
        dev::prefetch_tensormap(&tmv);
    }
    if (p.fuse_prefix_blocks == 0) dev::grid_dependency_wait();
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort;
    __shared__ int s_issued;
    __shared__ int s_rec_issued;
    uint8_t* stages = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* after = stages + (size_t)C::STAGES * C::STAGE;          // barriers, merge area
    const uint32_t full0 = dev::smem_addr(after);
    const uint32_t empty0 = full0 + 8 * C::STAGES;
    // one CTA per suffix: the prefix records' barrier and buffer follow the
    // stage barriers (rec_smem bytes of dynamic shared memory)
    const uint32_t rec_bar = empty0 + 8 * C::STAGES;
    float* rec_buf = reinterpret_cast<float*>(after + 16 * C::STAGES + 16);

    const int G = p.Hq / p.Hkv;
    const int gc = C::MMA ? G : C::GC;          // query heads this CTA serves
    const int chunks = G / gc;                  // head chunks per kv head
    int part = p.heads_fastest ? blockIdx.y : blockIdx.x;
    const int hc = p.heads_fastest ? blockIdx.x : blockIdx.y;
    // one kv head (or head chunk) per CTA, or HG neighbouring kv heads: kvh
    // is the first, h0 its first query head
    const int kvh = C::HG > 1 ? hc * C::HG : hc / chunks;
    const int h0 = C::HG > 1 ? kvh * G : kvh * G + (hc % chunks) * gc;
    const int s = blockIdx.z;
    // the producer's first 32 block ids, for the first block this CTA most
    // likely reads, fetched beside the context length
    const int pblk0_guess = p.fuse_prefix_blocks > 0 ? p.fuse_prefix_blocks
                            : p.prefix_parts > 0     ? -1
                                                     : part * p.part_group * p.part_blocks * C::PER;
    const int pre = (threadIdx.x >> 5) == C::NW ? table_entry_ahead(p, s, pblk0_guess) : 0;
    const int n = checked_len(p, s, C::PB);
    const int nphys_all = (n + C::PB - 1) / C::PB;
    const int nblk_all = (n + C::BS - 1) / C::BS;
    int blk0 = 0, nblk = nblk_all, nparts = 1;
    int q0 = part, nq = 1;                      // partitions (records) this CTA writes
    bool fuse_records = false;
    if (p.fuse_prefix_blocks > 0) {
        // A sequence whose table starts with row 0's prefix blocks (and that
        // holds the whole prefix) reads only its suffix here and merges the
        // prefix kernel's records in the epilogue; any other reads everything.
        const int pb = p.fuse_prefix_blocks;
        int irregular = 0;                      // the table loads do not wait for n
        for (int i = threadIdx.x; i < pb; i += blockDim.x)
            irregular |= p.block_tables[(size_t)s * p.MB + i] != p.block_tables[i];
        irregular = __syncthreads_or(irregular || n < pb * C::BS);
        if (!irregular) {
            blk0 = pb;
            nblk = nblk_all - pb;               // may be 0: the prefix alone
            fuse_records = true;
        }
    } else if (p.prefix_parts > 0) {
        // Shared-prefix decode: the grid covers the partitions past the
        // prefix (grid index i is partition prefix_parts + i); the prefix
        // kernel wrote partitions 0 .. prefix_parts-1 of every sequence.  A
        // sequence whose table does not start with row 0's prefix blocks, or
        // that is shorter than the prefix, is irregular: its first CTA covers
        // the prefix and partition prefix_parts in one record (partition 0)
        // and empties records 1 .. prefix_parts.
        const int k = p.prefix_parts;
        const int pb = k * p.part_blocks;
        int irregular = 0;
        if (part == 0) {
            irregular = n < pb * C::BS;
            for (int i = threadIdx.x; i < pb && !irregular; i += blockDim.x)
                irregular = p.block_tables[(size_t)s * p.MB + i] != p.block_tables[i];
            irregular = __syncthreads_or(irregular);
        }
        if (irregular) {
            for (int idx = threadIdx.x; idx < gc * k * (C::D + 1); idx += blockDim.x) {
                const int g = idx / (k * (C::D + 1)), rest = idx % (k * (C::D + 1));
                const int pp = 1 + rest / (C::D + 1), d = rest % (C::D + 1);
                const size_t row = ((size_t)s * p.Hq + h0 + g) * p.max_parts + pp;
                if (d == C::D) p.ws_ml[row] = make_float2(-INFINITY, 0.f);
                else p.ws_o[row * C::D + d] = 0.f;
            }
            nblk = min((k + 1) * p.part_blocks, nblk_all);   // blk0 = 0, record 0
        } else {
            part += k;
            blk0 = part * p.part_blocks;
            nblk = min(p.part_blocks, nblk_all - blk0);
            if (nblk <= 0) return;              // this sequence has fewer partitions
        }
        nparts = 2;                             // records always go through the workspace
    } else if (p.part_blocks > 0) {
        // grid index `part` covers partitions q0 .. q0 + part_group - 1
        q0 = part * p.part_group;
        blk0 = q0 * p.part_blocks;
        nblk = min(p.part_group * p.part_blocks, nblk_all - blk0);
        nparts = max(1, (nblk_all + p.part_blocks - 1) / p.part_blocks);
        nq = min(p.part_group, nparts - q0);
    }
    if (part > 0 && nblk <= 0) return;          // this sequence has fewer partitions
    nblk = max(nblk, 0);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the prefix records of a regular suffix arrive by a bulk copy the
    // producer issues after its last K/V copy (and after the prefix kernel)
    const bool rec_async = fuse_records && p.rec_smem > 0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::STAGES; ++i) {
            dev::mbar_init(full0 + 8 * i, 1);
            dev::mbar_init(empty0 + 8 * i, C::HG > 1 ? C::NW : 1);   // head groups: every warp
        }
        if (rec_async) dev::mbar_init(rec_bar, 1);
        dev::fence_mbar_init();
        s_abort = 0;
        s_issued = 0;
        s_rec_issued = 0;
    }
    __syncthreads();

    float* comb = reinterpret_cast<float*>(stages);
    float* cm = comb;
    float* cl = cm + C::NW * C::GC;
    float* co = cl + C::NW * C::GC;

    using State = typename std::conditional<C::MMA, MmaState<C>, SimtState<C>>::type;
    State st;
    if constexpr (GROUPED) {
        // Grouped partitions: the producer streams the blocks of all nq
        // partitions without a break; the consumers close each partition with
        // a warp merge through a dedicated area (the stages keep streaming)
        // and write its record, exactly as nq one-partition CTAs would.  With
        // head groups each warp holds a whole head's state and closes the
        // partition alone, through its own slice of that area.
        const int gh = gc;
        float* gm = reinterpret_cast<float*>(after + 16 * C::STAGES);
        float* gl = gm + C::NW * gh;
        float* go = gl + C::NW * gh;
        if (warp == C::NW) {
            int k = 0;
            produce<C>(&tmk, &tmv, p, p.block_tables + (size_t)s * p.MB, blk0, nblk,
                       min(nblk * C::PER, nphys_all - blk0 * C::PER), kvh, stages, full0, empty0,
                       &s_abort, &k, pblk0_guess, pre);
            if (lane == 0) s_issued = k;
        } else if constexpr (C::HG > 1) {
            // warp w: kv head kvh + w, its tiles in every stage
            const int hw = warp;
            mma_load_q<C>(st, p, s, h0 + hw * G, G);
            bool stop = false;
            for (int qq = 0; qq < nq && !stop; ++qq) {
                const int jb = qq * p.part_blocks, je = min(jb + p.part_blocks, nblk);
                for (int j = jb; j < je; ++j) {
                    const int stg = j % C::STAGES;
                    if (!dev::mbar_wait_bounded(full0 + 8 * stg, (j / C::STAGES) & 1)) {
                        if (lane == 0) { wait_timeout(p, 2); s_abort = 1; }
                        stop = true;
                        break;
                    }
                    uint8_t* kt = stages + (size_t)stg * C::STAGE + hw * C::PB * 128;
                    const int nvalid = min(C::BS, n - (blk0 + j) * C::BS);
                    mma_block<C>(st, kt, kt + C::TILE, nvalid, p.qk_scale);
                    __syncwarp();
                    if (lane == 0) dev::mbar_arrive(empty0 + 8 * stg);
                    if (*(volatile int*)&s_abort) { stop = true; break; }
                }
                if (stop) break;
                // this partition's record of the warp's query heads (the output
                // itself for a sequence of one partition: the merge skips it)
                mma_publish<C>(st, gm + hw * gh, gl + hw * gh, go + (size_t)hw * gh * C::D, 0, G, gh);
                __syncwarp();
                for (int idx = lane; idx < G * C::D; idx += 32) {
                    const int g = idx / C::D, d = idx % C::D;
                    const int h = h0 + hw * G + g;
                    const float O = go[((size_t)hw * gh + g) * C::D + d], L = gl[hw * gh + g];
                    if (nparts == 1) {
                        dev::store_out<C::QT>(p.out, ((size_t)s * p.Hq + h) * C::D + d,
                                              L == 0.f ? 0.f : (O / L) * p.v_scale);
                    } else {
                        const size_t row = ((size_t)s * p.Hq + h) * p.max_parts + q0 + qq;
                        p.ws_o[row * C::D + d] = O * p.v_scale;
                        if (d == 0) p.ws_ml[row] = make_float2(gm[hw * gh + g], L);
                    }
                }
                __syncwarp();
                mma_reset<C>(st);
            }
        } else {
            if constexpr (C::MMA) mma_load_q<C>(st, p, s, h0, G);
            else simt_load_q<C>(st, p, s, h0);
            bool stop = false;
            for (int qq = 0; qq < nq; ++qq) {
                const int jb = qq * p.part_blocks, je = min(jb + p.part_blocks, nblk);
                // this warp's blocks: j % NW == warp (the stage ring's owner rule)
                for (int j = jb + (warp - jb % C::NW + C::NW) % C::NW; j < je && !stop;
                     j += C::NW) {
                    const int stg = j % C::STAGES;
                    if (!dev::mbar_wait_bounded(full0 + 8 * stg, (j / C::STAGES) & 1)) {
                        if (lane == 0) { wait_timeout(p, 2); s_abort = 1; }
                        stop = true;
                        break;
                    }
                    uint8_t* kt = stages + (size_t)stg * C::STAGE;
                    const int nvalid = min(C::BS, n - (blk0 + j) * C::BS);
                    if constexpr (C::MMA)
                        mma_block<C>(st, kt, kt + C::TILE, nvalid, p.qk_scale);
                    else simt_block<C>(st, kt, kt + C::TILE, nvalid);
                    __syncwarp();
                    if (lane == 0) dev::mbar_arrive(empty0 + 8 * stg);
                    if (*(volatile int*)&s_abort) stop = true;
                }
                if constexpr (C::MMA) mma_publish<C>(st, gm, gl, go, warp, G, gh);
                else simt_publish<C>(st, gm, gl, go, warp);
                consumers_sync<C>();
                if (!*(volatile int*)&s_abort) {
                    for (int idx = threadIdx.x; idx < gh * C::D; idx += C::NW * 32) {
                        const int g = idx / C::D, d = idx % C::D;
                        float M = -INFINITY;
                        #pragma unroll
                        for (int w = 0; w < C::NW; ++w) M = fmaxf(M, gm[w * gh + g]);
                        float L = 0.f, O = 0.f;
                        if (M != -INFINITY) {
                            #pragma unroll
                            for (int w = 0; w < C::NW; ++w) {
                                const float f = exp2f(gm[w * gh + g] - M);
                                L = fmaf(f, gl[w * gh + g], L);
                                O = fmaf(f, go[(w * gh + g) * C::D + d], O);
                            }
                        }
                        const int h = h0 + g;
                        if (nparts == 1) {
                            dev::store_out<C::QT>(p.out, ((size_t)s * p.Hq + h) * C::D + d,
                                                  L == 0.f ? 0.f : (O / L) * p.v_scale);
                        } else {
                            const size_t row = ((size_t)s * p.Hq + h) * p.max_parts + q0 + qq;
                            p.ws_o[row * C::D + d] = O * p.v_scale;
                            if (d == 0) p.ws_ml[row] = make_float2(M, L);
                        }
                    }
                }
                // the merge area is free again; leave together on an abort
                if (consumers_sync_or<C>(stop || *(volatile int*)&s_abort)) break;
                if constexpr (C::MMA) mma_reset<C>(st);
                else simt_reset<C>(st);
            }
        }
        __syncthreads();
        dev::launch_dependents();
        if (s_abort && warp == C::NW && lane == 0) {
            // drain: every issued copy lands before the CTA leaves (bounded)
            const int issued = s_issued;
            for (int j = max(0, issued - C::STAGES); j < issued; ++j)
                dev::mbar_wait_bounded(full0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1);
        }
        return;
    }
    if (warp == C::NW) {
        int k = 0;
        const int32_t* bt_row = p.block_tables + (size_t)s * p.MB;
        const int nphys = min(nblk * C::PER, nphys_all - blk0 * C::PER);
        // a regular suffix's prefix records are fetched once the ring is first
        // full (the producer would wait for a free stage next anyway)
        const int first = rec_async ? min(nblk, C::STAGES) : nblk;
        produce<C>(&tmk, &tmv, p, bt_row, blk0, first, min(nphys, first * C::PER), kvh, stages,
                   full0, empty0, &s_abort, &k, pblk0_guess, pre);
        if (rec_async && lane == 0 && !*(volatile int*)&s_abort) {
            // [heads][max_parts][D] then [heads][max_parts], contiguous in the workspace
            dev::grid_dependency_wait();            // the prefix kernel has written them
            const int nh = C::HG * gc;
            const size_t row0 = ((size_t)s * p.Hq + h0) * p.max_parts;
            const uint32_t bo = (uint32_t)(nh * p.max_parts * C::D * 4);
            const uint32_t bm = (uint32_t)(nh * p.max_parts * 8);
            dev::mbar_arrive_expect_tx(rec_bar, bo + bm);
            dev::bulk_load(dev::smem_addr(rec_buf), p.ws_o + row0 * C::D, bo, rec_bar);
            dev::bulk_load(dev::smem_addr(rec_buf) + bo, p.ws_ml + row0, bm, rec_bar);
            s_rec_issued = 1;
        }
        __syncwarp();
        if (first < nblk && !*(volatile int*)&s_abort)
            produce<C>(&tmk, &tmv, p, bt_row, blk0 + first, nblk - first,
                       nphys - first * C::PER, kvh, stages, full0, empty0, &s_abort, &k);
        if (lane == 0) s_issued = k;
    } else {
        // one head per CTA: warp w takes stages w, w + NW, ...; head groups:
        // warp w takes every stage, and the tiles of kv head kvh + w in it
        const int hw = C::HG > 1 ? warp : 0;
        if constexpr (C::MMA) mma_load_q<C>(st, p, s, h0 + hw * G, G);
        else simt_load_q<C>(st, p, s, h0);
        for (int j = C::HG > 1 ? 0 : warp; j < nblk; j += C::HG > 1 ? 1 : C::NW) {
            const int stg = j % C::STAGES;
            if (!dev::mbar_wait_bounded(full0 + 8 * stg, (j / C::STAGES) & 1)) {
                if (lane == 0) { wait_timeout(p, 2); s_abort = 1; }
                break;
            }
            uint8_t* kt = stages + (size_t)stg * C::STAGE + hw * C::PB * 128;
            const int nvalid = min(C::BS, n - (blk0 + j) * C::BS);
            if constexpr (C::MMA)
                mma_block<C>(st, kt, kt + C::TILE, nvalid, p.qk_scale);
            else simt_block<C>(st, kt, kt + C::TILE, nvalid);
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(empty0 + 8 * stg);
            if (*(volatile int*)&s_abort) break;
        }
    }
    __syncthreads();                             // every stage consumed (or abort)
    dev::launch_dependents();                    // the merge kernel may start launching

    if (s_abort) {
        // Drain: wait (bounded) until every issued copy has landed, then leave.
        if (warp == C::NW && lane == 0) {
            const int issued = s_issued;
            for (int j = max(0, issued - C::STAGES); j < issued; ++j)
                dev::mbar_wait_bounded(full0 + 8 * (j % C::STAGES), (j / C::STAGES) & 1);
            if (s_rec_issued) dev::mbar_wait_bounded(rec_bar, 0);
        }
        return;
    }
    if (warp < C::NW) {
        if constexpr (C::MMA) mma_publish<C>(st, cm, cl, co, warp, G);
        else simt_publish<C>(st, cm, cl, co, warp);
    }
    if (p.fuse_prefix_blocks > 0) dev::grid_dependency_wait();   // the prefix records are written
    __syncthreads();

    // Shared-prefix records of this CTA's query heads, copied to shared memory
    // behind the warp-merge area with every load in flight at once (one round
    // trip instead of one per output element a thread writes).  They are
    // contiguous in the workspace: [heads][max_parts][D] and [heads][max_parts].
    const int nh = C::HG * gc;                  // query heads this CTA writes
    float* rec_o = rec_async ? rec_buf : comb + C::COMBINE_FLOATS;
    float2* rec_ml = reinterpret_cast<float2*>(rec_o + (size_t)nh * p.max_parts * C::D);
    // (staged: also room for the merge weights, nh * (NW + max_parts + 2) floats)
    const bool staged = fuse_records &&
                        (rec_async || (size_t)(C::COMBINE_FLOATS + nh * p.max_parts * (C::D + 2) +
                                               nh * (C::NW + p.max_parts + 2)) *
                                              4 <= (size_t)C::STAGES * C::STAGE);
    if (rec_async) {
        // issued by the producer after its last K/V copy; normally landed by now
        if (!dev::mbar_wait_bounded(rec_bar, 0)) {
            if (threadIdx.x == 0) wait_timeout(p, 19);
            return;
        }
    } else if (staged) {
        const size_t row0 = ((size_t)s * p.Hq + h0) * p.max_parts;
        const float4* src = reinterpret_cast<const float4*>(p.ws_o + row0 * C::D);
        float4* dst = reinterpret_cast<float4*>(rec_o);
        const int n4 = nh * p.max_parts * C::D / 4;
        constexpr int U = 4;
        for (int i0 = threadIdx.x; i0 < n4; i0 += U * C::THREADS) {
            float4 r[U];
            #pragma unroll
            for (int u = 0; u < U; ++u)
                if (i0 + u * C::THREADS < n4) r[u] = src[i0 + u * C::THREADS];
            #pragma unroll
            for (int u = 0; u < U; ++u)
                if (i0 + u * C::THREADS < n4) dst[i0 + u * C::THREADS] = r[u];
        }
        for (int i = threadIdx.x; i < nh * p.max_parts; i += C::THREADS) rec_ml[i] = p.ws_ml[row0 + i];
        __syncthreads();
    }

    // ---- merge the warps' states (and the prefix records) and write -----
    // Phase 1, one warp per query head row: lane i takes partial state i (the
    // consumer warps', or with head groups its warp's; then the prefix
    // records), and the warp reduces the common maximum M, the weights
    // 2^(m_i - M) and the sum L = sum of weight_i * l_i.  Phase 2, four
    // neighbouring output elements per thread: the weighted sum of the partial
    // outputs, with no exponential per element.  (The split-K identity: up to
    // rounding order the same as merging the states one after another.)
    const int nsrc = C::HG > 1 ? 1 : C::NW;     // partial states per head
    const int npre = fuse_records ? p.prefix_parts : 0;
    const int ncoef = nsrc + npre + 2;          // weights, then M and 1/L (0 for L = 0)
    float* coef = comb + C::COMBINE_FLOATS +
                  (staged && !rec_async ? (size_t)nh * p.max_parts * (C::D + 2) : 0);
    // partial state i of head row r (r = local query head: w * G + g with head groups)
    auto src_row = [&](int r, int i) { return C::HG > 1 ? (r / gc) * C::GC + r % gc : i * C::GC + r; };
    const size_t grow0 = ((size_t)s * p.Hq + h0) * p.max_parts;   // records of row 0 (global)
    auto src_ml = [&](int r, int i) -> float2 {
        if (i < nsrc) {
            const int q = src_row(r, i);
            return make_float2(cm[q], cl[q]);
        }
        const int pp = i - nsrc;
        return staged ? rec_ml[r * p.max_parts + pp] : p.ws_ml[grow0 + (size_t)r * p.max_parts + pp];
    };
    for (int r = warp; r < nh; r += C::THREADS / 32) {
        float M = -INFINITY;
        for (int i = lane; i < nsrc + npre; i += 32) M = fmaxf(M, src_ml(r, i).x);
        #pragma unroll
        for (int x = 16; x >= 1; x >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, x));
        float L = 0.f;
        float* c = coef + r * ncoef;
        for (int i = lane; i < nsrc + npre; i += 32) {
            const float2 ml = src_ml(r, i);
            const float e = M == -INFINITY ? 0.f : exp2f(ml.x - M);
            c[i] = e;
            L = fmaf(e, ml.y, L);
        }
        #pragma unroll
        for (int x = 16; x >= 1; x >>= 1) L += __shfl_xor_sync(0xffffffffu, L, x);
        if (lane == 0) {
            c[ncoef - 2] = M;
            c[ncoef - 1] = L == 0.f ? 0.f : 1.f / L;
            if (!fuse_records && !(nparts == 1 && !p.force_ws)) {
                const int h = C::HG > 1 ? h0 + (r / gc) * G + r % gc : h0 + r;
                p.ws_ml[((size_t)s * p.Hq + h) * p.max_parts + part] = make_float2(M, L);
            }
        }
    }
    __syncthreads();
    constexpr int D4 = C::D / 4;
    for (int idx = threadIdx.x; idx < nh * D4; idx += C::THREADS) {
        const int r = idx / D4, d = (idx % D4) * 4;
        const int h = C::HG > 1 ? h0 + (r / gc) * G + r % gc : h0 + r;
        const float* c = coef + r * ncoef;
        const float inv_l = c[ncoef - 1];
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < nsrc; ++i) {
            const float4 v = *reinterpret_cast<const float4*>(co + src_row(r, i) * C::D + d);
            O.x = fmaf(c[i], v.x, O.x);
            O.y = fmaf(c[i], v.y, O.y);
            O.z = fmaf(c[i], v.z, O.z);
            O.w = fmaf(c[i], v.w, O.w);
        }
        const size_t o0 = ((size_t)s * p.Hq + h) * C::D + d;
        if (fuse_records) {
            // the prefix records' o is already times v_scale
            float4 Op = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int pp = 0; pp < npre; ++pp) {
                const float w = c[nsrc + pp];
                float4 v;
                if (staged) {
                    v = *reinterpret_cast<const float4*>(rec_o + ((size_t)r * p.max_parts + pp) * C::D + d);
                } else {
                    const float* g = p.ws_o + (grow0 + (size_t)r * p.max_parts + pp) * C::D + d;
                    v = make_float4(g[0], g[1], g[2], g[3]);
                }
                Op.x = fmaf(w, v.x, Op.x);
                Op.y = fmaf(w, v.y, Op.y);
                Op.z = fmaf(w, v.z, Op.z);
                Op.w = fmaf(w, v.w, Op.w);
            }
            dev::store_out<C::QT>(p.out, o0 + 0, fmaf(O.x, p.v_scale, Op.x) * inv_l);
            dev::store_out<C::QT>(p.out, o0 + 1, fmaf(O.y, p.v_scale, Op.y) * inv_l);
            dev::store_out<C::QT>(p.out, o0 + 2, fmaf(O.z, p.v_scale, Op.z) * inv_l);
            dev::store_out<C::QT>(p.out, o0 + 3, fmaf(O.w, p.v_scale, Op.w) * inv_l);
        } else if (nparts == 1 && !p.force_ws) {
            const float f = inv_l * p.v_scale;
            dev::store_out<C::QT>(p.out, o0 + 0, O.x * f);
            dev::store_out<C::QT>(p.out, o0 + 1, O.y * f);
            dev::store_out<C::QT>(p.out, o0 + 2, O.z * f);
            dev::store_out<C::QT>(p.out, o0 + 3, O.w * f);
        } else {
            const size_t row = ((size_t)s * p.Hq + h) * p.max_parts + part;
            float* w = p.ws_o + row * C::D + d;
            w[0] = O.x * p.v_scale;
            w[1] = O.y * p.v_scale;
            w[2] = O.z * p.v_scale;
            w[3] = O.w * p.v_scale;
        }
    }
}

// ------------------------------------------------------ balanced kernel
// Persistent, work-balanced variant ("stream-K").  Items are (sequence, kv
// head [, head chunk]) pairs, laid end to end in one global block space of W
// blocks (item i = s * HC + hc holds ceil(n_s / bs) blocks).  CTA c of a
// grid sized to the GPU's resident capacity takes blocks [c*W/grid,
// (c+1)*W/grid): equal work to one block, no atomics, no per-call state.
// Its producer walks that range item by item without draining the stage ring
// between items, and publishes each piece (the part of one item inside the
// range) through a small ring of descriptors.  Consumers finish a piece with
// a two-phase rendezvous on mbarriers (bounded waits): a piece that is a whole
// item is written out directly; a piece of a split item is written as a
// partial at row (item + c) * gc + g, and the item's first / last piece record
// which CTAs hold it, for decode_merge.
constexpr int kItemQ = 4;

struct PieceDesc {
    int s, hc, off, take, nblk, n, k0, end, fold;
};

template <class C>
struct BalancedSmem {
    static constexpr int STAGES_RAW = 64 * 1024 / C::STAGE;  // 3 CTAs per SM fit
    // a multiple of NW: each stage has a single consumer warp (see Cfg)
    static constexpr int STAGES_CLAMPED = STAGES_RAW < C::NW ? C::NW : (STAGES_RAW > 32 ? 32 : STAGES_RAW);
    static constexpr int STAGES = STAGES_CLAMPED / C::NW * C::NW;
    static_assert(STAGES % C::NW == 0, "each stage must have a single consumer warp");
    // the warp-merge area holds NW * gc * (D + 2) floats, gc = query heads per
    // item (known at launch); it follows the barriers
    static constexpr size_t FIXED = 1024 + size_t(STAGES) * C::STAGE +
                                    8 * (2 * STAGES + 2 * kItemQ + 2);
    static size_t bytes(int gc) { return FIXED + size_t(C::NW) * gc * (C::D + 2) * 4; }
};

// Work of each of sequence s's items in the balanced grid's block space.
// Split pieces: its blocks.  Whole items: its blocks past a shared prefix it
// is expected to skip (long enough to hold it; the producer checks the table
// itself, so a wrong guess costs balance, never correctness), plus one for
// the item's own start-up and epilogue (an item with no block still needs its
// output written).
template <class C>
__device__ __forceinline__ int blocks_of(const Params& p, int s) {
    const int n = checked_len(p, s, C::BS);
    const int nb = (n + C::BS - 1) / C::BS;
    if (!p.whole_items) return nb;
    const int pb = p.fuse_prefix_blocks;
    return (pb > 0 && n >= pb * C::BS ? nb - pb : nb) + 1;
}


// The configuration of the balanced kernel: the same tile shapes, a deeper ring.
template <class C>
struct Balanced : C {
    static constexpr int STAGES = BalancedSmem<C>::STAGES;
};

template <class C0>
__global__ void __launch_bounds__(C0::THREADS, 3)
decode_balanced(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                const Params p) {
    // Launched as a dependent of the kernel before it.  Whole items of the
    // shared-prefix decode read nothing that kernel (the prefix kernel) writes
    // until they fold its records in, so they wait there and stream their
    // suffixes meanwhile; everything the kernels before that one wrote was
    // complete when its CTAs let this grid start.
    if (!p.whole_items) dev::grid_dependency_wait();
    using B = BalancedSmem<C0>;
    using C = Balanced<C0>;
    constexpr int STAGES = B::STAGES;
    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_abort, s_issued, s_found, s_s0, s_hc0, s_off0;
    __shared__ long long s_red[C::NW + 1];
    __shared__ PieceDesc s_ring[kItemQ];
    uint8_t* stages = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* after = stages + (size_t)STAGES * C::STAGE;                  // barriers, merge area
    const uint32_t full0 = dev::smem_addr(after);
    const uint32_t empty0 = full0 + 8 * STAGES;
    const uint32_t ifull0 = empty0 + 8 * STAGES;
    const uint32_t iempty0 = ifull0 + 8 * kItemQ;
    const uint32_t rdv_pub = iempty0 + 8 * kItemQ;     // consumers published their states
    const uint32_t rdv_done = rdv_pub + 8;              // consumers finished the combine
    float* comb = reinterpret_cast<float*>(after +
                                           8 * (2 * STAGES + 2 * kItemQ + 2));

    const int G = p.Hq / p.Hkv;
    const int gc = C::MMA ? G : C::GC;
    const int chunks = G / gc;
    const int HC = p.Hkv * chunks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Whole items are striped by head: the grid is HC CTAs per group, group g
    // takes a contiguous run of sequences of about equal total work and CTA
    // (g, hc) serves head hc of each.  The heads of a sequence have the same
    // length, so a group's CTAs keep pace and read each block's head rows
    // (neighbours in memory) at about the same time.  The split mode spreads
    // (sequence, head) items over single CTAs.
    const bool whole = p.whole_items != 0;
    const int span = whole ? 1 : HC;                    // items per sequence in the space
    const long long units = whole ? (long long)(gridDim.x / HC) : (long long)gridDim.x;
    const long long unit = whole ? (long long)(blockIdx.x / HC) : (long long)blockIdx.x;
    const int my_hc = whole ? (int)(blockIdx.x % HC) : 0;

    // ---- W and this CTA's block range --------------------------------------
    long long acc = 0;
    for (int s = threadIdx.x; s < p.S; s += C::THREADS) acc += (long long)blocks_of<C>(p, s) * span;
    #pragma unroll
    for (int x = 16; x > 0; x >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
    if (lane == 0) s_red[warp] = acc;
    if (threadIdx.x == 0) s_found = 0;
    __syncthreads();
    long long W = 0;
    #pragma unroll
    for (int w = 0; w <= C::NW; ++w) W += s_red[w];
    // With fewer blocks than CTAs (groups) only the first W work, so every
    // working share is non-empty and an item's pieces sit on consecutive CTAs.
    const long long nctas = W < units ? W : units;
    if (unit >= nctas) return;                          // CTA-uniform: no work
    const long long b0 = unit * W / nctas;
    const long long b1 = (unit + 1) * W / nctas;
    __syncthreads();                                    // s_red is reused below
    long long R = 0;
    for (int base = 0; base < p.S; base += C::THREADS) {
        const int s = base + threadIdx.x;
        const int nb = s < p.S ? blocks_of<C>(p, s) : 0;
        const long long v = (long long)nb * span;
        long long inc = v;
        #pragma unroll
        for (int x = 1; x < 32; x <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, inc, x);
            if (lane >= x) inc += y;
        }
        if (lane == 31) s_red[warp] = inc;
        __syncthreads();
        long long woff = 0, tile = 0;
        #pragma unroll
        for (int w = 0; w <= C::NW; ++w) {
            if (w < warp) woff += s_red[w];
            tile += s_red[w];
        }
        const long long ex = R + woff + inc - v;
        if (v > 0 && ex <= b0 && b0 < ex + v) {
            const long long rel = b0 - ex;
            s_s0 = s;
            s_hc0 = (int)(rel / nb);
            s_off0 = (int)(rel % nb);
            s_found = 1;
        }
        R += tile;
        __syncthreads();
        if (s_found || R > b0) break;                  // CTA-uniform
    }

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            dev::mbar_init(full0 + 8 * i, 1);
            dev::mbar_init(empty0 + 8 * i, 1);
        }
        for (int i = 0; i < kItemQ; ++i) {
            dev::mbar_init(ifull0 + 8 * i, 1);
            dev::mbar_init(iempty0 + 8 * i, C::NW);
        }
        dev::mbar_init(rdv_pub, C::NW);
        dev::mbar_init(rdv_done, C::NW);
        dev::fence_mbar_init();
        s_abort = 0;
        s_issued = 0;
    }
    if (warp == C::NW && lane == 0) {
        dev::prefetch_tensormap(&tmk);
        dev::prefetch_tensormap(&tmv);
    }
    __syncthreads();

    using State = typename std::conditional<C::MMA, MmaState<C>, SimtState<C>>::type;
    State st;
    if (warp == C::NW) {
        // ---------------------------------------------------------- producer
        int s = s_s0, hc = s_hc0, off = s_off0, k = 0, ci = 0;
        long long b = b0;
        bool stop = !s_found;
        auto publish = [&](const PieceDesc& d) {
            int bad = 0;
            if (lane == 0) {
                const int slot = ci % kItemQ;
                if (ci >= kItemQ &&
                    !dev::mbar_wait_bounded(iempty0 + 8 * slot, ((ci / kItemQ) & 1) ^ 1)) {
                    wait_timeout(p, 3);
                    s_abort = 1;
                    bad = 1;
                } else {
                    s_ring[slot] = d;
                    dev::mbar_arrive(ifull0 + 8 * slot);
                }
            }
            return __shfl_sync(0xffffffffu, bad, 0) != 0;
        };
        if (whole) {
            // Whole items: this CTA takes head my_hc of the sequences that
            // start inside [b0, b1); the sequence holding b0 is its group's
            // only if it starts there.
            hc = my_hc;
            b -= off;
            if (!stop && off > 0) {
                b += blocks_of<C>(p, s);
                ++s;
            }
            const int pb = p.fuse_prefix_blocks;
            int reg_s = -1, reg = 0;                   // regularity of sequence reg_s
            while (!stop && b < b1 && s < p.S) {
                const int n = checked_len(p, s, C::BS);
                const int nb = (n + C::BS - 1) / C::BS;
                if (pb > 0 && s != reg_s) {
                    // regular: long enough, and its table starts with row 0's prefix blocks
                    int diff = n < pb * C::BS;
                    for (int i = lane; i < pb && !diff; i += 32)
                        diff = __ldg(p.block_tables + (size_t)s * p.MB + i) != __ldg(p.block_tables + i);
                    reg = !__any_sync(0xffffffffu, diff);
                    reg_s = s;
                }
                const int blk0 = pb > 0 && reg ? pb : 0;
                PieceDesc d{s, hc, blk0, nb - blk0, nb, n, k, 0, blk0 > 0};
                if (publish(d)) break;
                {
                    // the consumers load this item's query rows when they reach
                    // it: have them in L2 by then
                    constexpr int QB = C::QT == PA_F32 ? 4 : 2;
                    const int hq0 = (hc / chunks) * G + (hc % chunks) * gc;
                    const char* qrow = static_cast<const char*>(p.q) +
                                       ((size_t)s * p.Hq + hq0) * C::D * QB;
                    for (int i = lane; i < (gc * C::D * QB + 127) / 128; i += 32)
                        dev::prefetch_l2(qrow + (size_t)i * 128);
                }
                produce<C>(&tmk, &tmv, p, p.block_tables + (size_t)s * p.MB, blk0, nb - blk0,
                            nb - blk0, hc / chunks, stages, full0, empty0, &s_abort, &k);
                if (*(volatile int*)&s_abort) break;
                b += blocks_of<C>(p, s);
                ++ci;
                ++s;
            }
        } else {
            while (!stop && b < b1 && s < p.S) {
                const int n = checked_len(p, s, C::BS);
                const int nb = (n + C::BS - 1) / C::BS;
                if (nb > off) {
                    const int take = (int)min((long long)(nb - off), b1 - b);
                    PieceDesc d{s, hc, off, take, nb, n, k, 0, 0};
                    if (publish(d)) break;
                    produce<C>(&tmk, &tmv, p, p.block_tables + (size_t)s * p.MB, off, take,
                                take, hc / chunks, stages, full0, empty0, &s_abort, &k);
                    if (*(volatile int*)&s_abort) break;
                    b += take;
                    ++ci;
                }
                off = 0;
                if (++hc == HC) { hc = 0; ++s; }
            }
        }
        if (!*(volatile int*)&s_abort) {
            PieceDesc d{0, 0, 0, 0, 0, 0, k, 1, 0};
            publish(d);
        }
        if (lane == 0) s_issued = k;
    } else {
        // --------------------------------------------------------- consumers
        float* cm = comb;                              // stride gc (heads per item)
        float* cl = cm + C::NW * gc;
        float* co = cl + C::NW * gc;
        bool records_ready = false;
        for (int ci = 0;; ++ci) {
            const int slot = ci % kItemQ;
            if (!dev::mbar_wait_bounded(ifull0 + 8 * slot, (ci / kItemQ) & 1)) {
                if (lane == 0) { wait_timeout(p, 4); s_abort = 1; }
                break;
            }
            const PieceDesc d = s_ring[slot];
            if (d.end) break;
            const int h0 = (d.hc / chunks) * G + (d.hc % chunks) * gc;
            if constexpr (C::MMA) mma_load_q<C>(st, p, d.s, h0, G);
            else simt_load_q<C>(st, p, d.s, h0);
            unsigned bad = 0;
            // block k goes to warp k % NW (not by its place in the piece), so a
            // stage, used by blocks k = stage (mod STAGES), keeps a single consumer
            const int jj0 = ((warp - d.k0) % C::NW + C::NW) % C::NW;
            for (int jj = jj0; jj < d.take; jj += C::NW) {
                const int k = d.k0 + jj;
                const int stg = k % STAGES;
                if (!dev::mbar_wait_bounded(full0 + 8 * stg, (k / STAGES) & 1)) { bad = 2; break; }
                uint8_t* kt = stages + (size_t)stg * C::STAGE;
                const int nvalid = min(C::BS, d.n - (d.off + jj) * C::BS);
                if constexpr (C::MMA)
                    mma_block<C>(st, kt, kt + C::TILE, nvalid, p.qk_scale);
                else simt_block<C>(st, kt, kt + C::TILE, nvalid);
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(empty0 + 8 * stg);
            }
            if (!bad) {
                if constexpr (C::MMA) mma_publish<C>(st, cm, cl, co, warp, G, gc);
                else simt_publish<C>(st, cm, cl, co, warp, gc);
                __syncwarp();
                if (lane == 0) dev::mbar_arrive(rdv_pub);
                if (!dev::mbar_wait_bounded(rdv_pub, ci & 1)) bad = 5;
            }
            if (bad) {
                if (lane == 0) { wait_timeout(p, bad); s_abort = 1; }
                break;
            }
            // ---- combine the four warps' states for this piece -----------
            const int item = d.s * HC + d.hc;
            const bool whole = p.whole_items != 0;
            const bool first = whole || d.off == 0, last = whole || d.off + d.take == d.nblk;
            const int piece = item + blockIdx.x;
            if (d.fold) {
                if (!records_ready) {
                    dev::grid_dependency_wait();        // the prefix kernel wrote them
                    records_ready = true;
                }
                fold_item<C>(p, d.s, h0, gc, cm, cl, co);
            } else
            for (int idx = threadIdx.x; idx < gc * C::D; idx += C::NW * 32) {
                const int g = idx / C::D, dd = idx % C::D;
                float M = -INFINITY;
                #pragma unroll
                for (int w = 0; w < C::NW; ++w) M = fmaxf(M, cm[w * gc + g]);
                float L = 0.f, O = 0.f;
                if (M != -INFINITY) {
                    #pragma unroll
                    for (int w = 0; w < C::NW; ++w) {
                        const float f = exp2f(cm[w * gc + g] - M);
                        L = fmaf(f, cl[w * gc + g], L);
                        O = fmaf(f, co[(w * gc + g) * C::D + dd], O);
                    }
                }
                if (first && last) {
                    dev::store_out<C::QT>(p.out, ((size_t)d.s * p.Hq + h0 + g) * C::D + dd,
                                          L == 0.f ? 0.f : (O / L) * p.v_scale);
                } else {
                    const size_t row = (size_t)piece * gc + g;
                    if ((int64_t)row < p.ws_rows) {
                        p.ws_o[row * C::D + dd] = O * p.v_scale;
                        if (dd == 0) p.ws_ml[row] = make_float2(M, L);
                    } else if (dd == 0) {
                        dev::raise_error(p.err, PA_DEV_BAD_PIECES);
                    }
                }
            }
            if (threadIdx.x == 0 && !whole) {
                if (first) p.ws_item[item].x = blockIdx.x;
                if (last) p.ws_item[item].y = blockIdx.x;
            }
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(rdv_done);
            if (!dev::mbar_wait_bounded(rdv_done, ci & 1)) {
                if (lane == 0) { wait_timeout(p, 6); s_abort = 1; }
                break;
            }
            if (lane == 0) dev::mbar_arrive(iempty0 + 8 * slot);
        }
    }
    __syncthreads();
    dev::launch_dependents();
    if (s_abort && warp == C::NW && lane == 0) {
        const int issued = s_issued;
        for (int j = max(0, issued - STAGES); j < issued; ++j)
            dev::mbar_wait_bounded(full0 + 8 * (j % STAGES), (j / STAGES) & 1);
    }
}

// Merge split-K partials: out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// A CTA of NWARPS warps serves NWARPS / wph query heads of one sequence; the
// wph warps of a head split its partitions, and each lane holds D/32 dims, so
// every partial row is one coalesced load.  8 warps by default; 32 for long
// contexts, whose hundreds of partials per head would otherwise be a chain of
// dependent loads per warp.  Launched as a programmatic dependent of the
// partition kernel: it waits for that grid's memory before reading.
constexpr int kMergeWarps = 8;
constexpr int kMergeWarpsLong = 32;

template <int QT, int D, int NWARPS>
__global__ void __launch_bounds__(NWARPS * 32) decode_merge(const Params p, int wph) {
    constexpr int DL = D / 32;                        // dims per lane
    __shared__ float s_max[NWARPS];
    __shared__ float s_l[NWARPS];
    __shared__ __align__(16) float s_o[NWARPS][D];
    __shared__ int s_live[NWARPS];
    dev::grid_dependency_wait();
    const int hpc = NWARPS / wph;                // heads per CTA
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hl = warp / wph, sub = warp % wph;
    const int h = blockIdx.x * hpc + hl, s = blockIdx.y;
    const bool head_ok = h < p.Hq;
    int n = p.context_lens[s];
    n = max(0, min(n, min(p.max_ctx, p.MB * p.bs)));
    // pieces of this head: count and first row (rows of consecutive pieces
    // are `stride` apart)
    int count = 0;
    size_t row0 = 0, stride = 1;
    if (p.balanced) {
        if (n == 0) {                                 // no CTA saw this sequence
            for (int idx = threadIdx.x; idx < hpc * D; idx += blockDim.x) {
                const int head = blockIdx.x * hpc + idx / D;
                if (head < p.Hq) dev::store_out<QT>(p.out, ((size_t)s * p.Hq + head) * D + idx % D, 0.f);
            }
            return;                                   // CTA-uniform
        }
        // piece c of item i sits at row (i + c) * gc + g, for c in [first CTA, last CTA]
        const int gc = p.gc;
        const int HC = p.Hq / gc;
        const int item = s * HC + (head_ok ? h : 0) / gc;
        const int2 fl = p.ws_item[item];
        count = fl.y - fl.x + 1;
        const bool sane = fl.x >= 0 && count >= 1 &&
                          (int64_t)(item + fl.y + 1) * gc <= p.ws_rows;
        if (!sane) {                                  // never follow a bad record
            if (head_ok && sub == 0 && lane == 0) dev::raise_error(p.err, PA_DEV_BAD_PIECES);
            count = 0;
        }
        row0 = sane ? (size_t)(item + fl.x) * gc + (head_ok ? h : 0) % gc : 0;
        stride = (size_t)gc;
    } else {
        count = min(p.max_parts, (n + p.part_tokens - 1) / p.part_tokens);
        if (count <= 1 && !p.force_ws) return;        // CTA-uniform: written by the partition kernel
        row0 = ((size_t)s * p.Hq + (head_ok ? h : 0)) * p.max_parts;
        stride = 1;
    }
    // count <= 1: written by the partition kernel, unless every record goes
    // through the workspace (then count 0, an empty sequence, writes zeros)
    const bool live = head_ok && (count > 1 || (p.force_ws && !p.balanced));
    if (sub == 0) s_live[hl] = live ? 1 : 0;

    float mx = -INFINITY;
    if (live)
        for (int i = sub * 32 + lane; i < count; i += wph * 32) mx = fmaxf(mx, p.ws_ml[row0 + i * stride].x);
    #pragma unroll
    for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
    if (lane == 0) s_max[warp] = mx;
    __syncthreads();
    float M = -INFINITY;
    for (int w = hl * wph; w < (hl + 1) * wph; ++w) M = fmaxf(M, s_max[w]);

    float L = 0.f, o[DL];
    #pragma unroll
    for (int k = 0; k < DL; ++k) o[k] = 0.f;
    if (live) {
        #pragma unroll 4
        for (int i = sub; i < count; i += wph) {
            const size_t row = row0 + i * stride;
            const float2 ml = p.ws_ml[row];
            const float f = exp2f(ml.x - M);
            L = fmaf(f, ml.y, L);
            const float* src = p.ws_o + row * D + lane * DL;
            if constexpr (DL % 4 == 0) {
                #pragma unroll
                for (int k = 0; k < DL; k += 4) {
                    const float4 v = *reinterpret_cast<const float4*>(src + k);
                    o[k] = fmaf(f, v.x, o[k]); o[k + 1] = fmaf(f, v.y, o[k + 1]);
                    o[k + 2] = fmaf(f, v.z, o[k + 2]); o[k + 3] = fmaf(f, v.w, o[k + 3]);
                }
            } else {
                #pragma unroll
                for (int k = 0; k < DL; ++k) o[k] = fmaf(f, src[k], o[k]);
            }
        }
    }
    if (lane == 0) s_l[warp] = L;
    #pragma unroll
    for (int k = 0; k < DL; ++k) s_o[warp][lane * DL + k] = o[k];
    __syncthreads();
    for (int idx = threadIdx.x; idx < hpc * D; idx += blockDim.x) {
        const int hh = idx / D, d = idx % D;
        const int head = blockIdx.x * hpc + hh;
        if (head >= p.Hq || !s_live[hh]) continue;   // not split: already written
        float Lt = 0.f, Ot = 0.f;
        for (int w = hh * wph; w < (hh + 1) * wph; ++w) {
            Lt += s_l[w];
            Ot += s_o[w][d];
        }
        dev::store_out<QT>(p.out, ((size_t)s * p.Hq + head) * D + d, Lt == 0.f ? 0.f : Ot / Lt);
    }
}

}  // namespace dec
}  // namespace pa
