// Host side of pa_decode: argument checks, tensor maps over the paged caches,
// split-K partitioning, kernel selection and launches.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "decode_launch.h"
#include "pa_internal.h"
#include "tma_host.h"

namespace pa {
namespace {

// pa_decode_select bits: 1 = CUDA-core consumer only, 2 = L2 evict-first
// hint on K/V loads, 4 = partition-major grid (kv heads of a partition side
// by side), 8 = group split-K partitions three to a CTA whenever there are
// several (a test hook for the grouped path at small sizes), 16 = shared-prefix
// decode with the persistent whole-item grid for the suffixes instead of one
// CTA per (sequence, kv head) suffix, 32 = one kv head per CTA everywhere (no
// head groups), 64 = pa_prefill on clusters of two CTAs, one per query tile of
// a pair (cta_group::2); the default is 4.
std::atomic<int> g_select{4};

// Plain split-K with short partitions: one CTA streams g consecutive
// partitions (each still its own record).  g minimises a simple model of
// the grid's time for equal-length sequences: the number of full waves of
// resident CTAs (3 per SM; a part-filled last wave costs nearly a whole
// one, since a lone CTA cannot pull its SM's share of HBM) times what a
// CTA streams plus its start-up and drain (about 6 us on the 4 x 100k
// workload, some 160 KB of a CTA's streaming).  Ties go to the larger g,
// the fewer CTAs.
// units: CTAs one partition per CTA would need per partition index (sequences
// x kv heads x head chunks); part_bytes: K/V bytes of one partition of one kv
// head.  Partitions of 512 KB or more are long enough on their own: g = 1.
int plan_part_group(int64_t units, int64_t max_parts, int64_t part_bytes, int num_sms,
                    int heads_per_cta = 1) {
    if (max_parts <= 1 || part_bytes / heads_per_cta >= (512 << 10)) return 1;
    const int64_t slots = 3LL * (num_sms > 0 ? num_sms : 148);
    double best = 0.0;
    int group = 1;
    for (int64_t g = 1; g <= std::min<int64_t>(max_parts, 4096); ++g) {
        const int64_t waves = (units * ((max_parts + g - 1) / g) + slots - 1) / slots;
        const double t = (double)waves * (double)(g * part_bytes + (160 << 10));
        if (g == 1 || t <= best) {
            best = t;
            group = (int)g;
        }
    }
    return group;
}

// Four kv heads per CTA (head groups) for the partition kernel: the
// tensor-core consumer, Hkv a multiple of 4, a stage of the four heads' K and
// V at most 32 KB, and select bit 32 off.  (The callers add the paths that
// keep one head: the balanced grid and the shared-prefix passes.)
bool decode_heads_per_cta(bool use_mma, int stage_tokens, int D, pa_dtype cache_dt, int Hkv,
                          int sel) {
    return use_mma && 2 * 4 * stage_tokens * D * elem_size(cache_dt) <= 32 * 1024 &&
           Hkv % 4 == 0 && !(sel & 32);
}

// SMs of the current device (cached per device; 148 if the query fails).
int sm_count() {
    static std::atomic<int> sms[256] = {};      // threads may race to fill an entry: same value
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 148;
    int n = sms[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return 148;
        sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Launched as a programmatic dependent of the partition kernel so its launch
// overlaps that grid's last wave (it waits for the grid's memory itself).
template <int QT, int D, int NW>
cudaError_t launch_merge_t(const dec::Params& p, int wph, dim3 grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(NW * 32);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, dec::decode_merge<QT, D, NW>, p, wph);
    if (e == cudaSuccess) note_launch();
    return e;
}

template <int QT, int D>
cudaError_t launch_merge_w(const dec::Params& p, int nw, int wph, dim3 grid, cudaStream_t st) {
    if (nw == dec::kMergeWarpsLong) return launch_merge_t<QT, D, dec::kMergeWarpsLong>(p, wph, grid, st);
    return launch_merge_t<QT, D, dec::kMergeWarps>(p, wph, grid, st);
}

template <int QT>
cudaError_t launch_merge_q(const dec::Params& p, int D, int nw, int wph, dim3 grid,
                           cudaStream_t st) {
    switch (D) {
    case 64: return launch_merge_w<QT, 64>(p, nw, wph, grid, st);
    case 128: return launch_merge_w<QT, 128>(p, nw, wph, grid, st);
    case 256: return launch_merge_w<QT, 256>(p, nw, wph, grid, st);
    }
    return cudaErrorNotSupported;
}

// Warps per head: enough to split a sequence's partitions (8 partitions a
// warp or fewer), at most the CTA's warps: 8, or 32 past 64 partitions.
cudaError_t launch_merge(const dec::Params& p, pa_dtype qt, int D, int Hq, int S,
                         cudaStream_t st) {
    const int nw = !p.balanced && p.max_parts > 64 ? dec::kMergeWarpsLong : dec::kMergeWarps;
    int wph = 1;
    if (p.balanced) wph = 2;     // pieces per item: about (item blocks / CTA range) + 1
    else while (wph < nw && p.max_parts > 8 * wph) wph *= 2;
    const int hpc = nw / wph;
    const dim3 grid((unsigned)((Hq + hpc - 1) / hpc), (unsigned)S);
    switch (qt) {
    case PA_F32: return launch_merge_q<PA_F32>(p, D, nw, wph, grid, st);
    case PA_F16: return launch_merge_q<PA_F16>(p, D, nw, wph, grid, st);
    case PA_BF16: return launch_merge_q<PA_BF16>(p, D, nw, wph, grid, st);
    default: return cudaErrorNotSupported;
    }
}

int64_t parts_for(int max_ctx, int partition) {
    if (partition <= 0 || max_ctx <= partition) return 1;
    return ((int64_t)max_ctx + partition - 1) / partition;
}

bool is_pow2_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

// The shape and dtype rules every decode launch obeys (pa_decode and the
// plan query pa_decode_partition_group share them, so the query never
// describes a launch that pa_decode would refuse).
pa_status check_decode_shape(pa_dtype q_dt, pa_dtype cache_dt, int S, int Hq, int Hkv, int D,
                             int bs, int max_ctx, int partition) {
    if (!valid_dtype(q_dt) || !valid_dtype(cache_dt)) return fail(PA_ERR_INVALID_ARG, "bad dtype");
    if (S < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_ctx < 0 || partition < PA_PARTITION_BALANCED)
        return fail(PA_ERR_INVALID_ARG, "negative or zero size");
    if (Hq % Hkv) return fail(PA_ERR_INVALID_ARG, "Hq (%d) is not a multiple of Hkv (%d)", Hq, Hkv);
    if (!(bs == 8 || bs == 16 || bs == 32))
        return fail(PA_ERR_UNSUPPORTED, "block size %d (supported: 8, 16, 32)", bs);
    if (partition != PA_PARTITION_BALANCED && partition % bs)
        return fail(PA_ERR_INVALID_ARG, "partition %d is not a multiple of bs", partition);
    const bool pair_ok = (cache_dt == q_dt && cache_dt != PA_FP8_E4M3) ||
                         (cache_dt == PA_FP8_E4M3 && (q_dt == PA_F16 || q_dt == PA_BF16));
    if (!pair_ok) return fail(PA_ERR_UNSUPPORTED, "cache dtype %d with q dtype %d", cache_dt, q_dt);
    const int row = D * elem_size(cache_dt);
    if (!((D == 64 || D == 128 || D == 256) && (row == 128 || row == 256 || row == 512)))
        return fail(PA_ERR_UNSUPPORTED, "head dim %d with this cache dtype", D);
    if (!is_pow2_group(Hq / Hkv)) return fail(PA_ERR_UNSUPPORTED, "group size %d", Hq / Hkv);
    return PA_OK;
}

}  // namespace
}  // namespace pa

using namespace pa;

// Balanced mode layout: [items] int2 (first, last CTA), 16-byte aligned, then
// [pieces * gc] float2 (m, l), then [pieces * gc * D] float (o), with
// items = S * HC, pieces = items + kMaxBalancedCtas, items * gc = S * Hq.
static size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

static size_t balanced_bytes(int S, int Hq, int D, int gc) {
    const size_t items = (size_t)S * (Hq / gc);
    const size_t rows = (items + dec::kMaxBalancedCtas) * gc;
    return align16(items * sizeof(int2)) + align16(rows * sizeof(float2)) + rows * sizeof(float) * D;
}

extern "C" pa_status pa_decode_workspace_size(int S, int Hq, int D, int max_ctx, int partition,
                                              size_t* bytes) {
    clear_error();
    if (!bytes) return fail(PA_ERR_INVALID_ARG, "bytes is NULL");
    if (S < 0 || Hq <= 0 || D <= 0 || max_ctx < 0 || partition < PA_PARTITION_BALANCED)
        return fail(PA_ERR_INVALID_ARG, "negative or zero size");
    if (partition == PA_PARTITION_BALANCED) {
        // the bound over every heads-per-item value (gc divides Hq, gc <= 16)
        size_t mx = 0;
        for (int gc = 1; gc <= 16 && gc <= Hq; gc *= 2)
            if (Hq % gc == 0 && balanced_bytes(S, Hq, D, gc) > mx) mx = balanced_bytes(S, Hq, D, gc);
        *bytes = mx;
        return PA_OK;
    }
    const int64_t mp = parts_for(max_ctx, partition);
    *bytes = mp <= 1 ? 0 : (size_t)S * Hq * mp * (sizeof(float) * 2 + sizeof(float) * D);
    return PA_OK;
}

extern "C" pa_status pa_decode_suggest_partition(int S, int Hkv, int bs,
                                                 const int32_t* context_lens_host, int* partition) {
    clear_error();
    if (!partition || (S > 0 && !context_lens_host) || S < 0 || Hkv <= 0 ||
        !(bs == 8 || bs == 16 || bs == 32))
        return fail(PA_ERR_INVALID_ARG, "bad arguments");
    // Enough CTAs for several waves on 148 SMs (3 resident per SM) so the last
    // wave is short, with partitions as long as that allows (each CTA pays a
    // start-up and drain of a few microseconds) and no shorter than 256 tokens.
    const int64_t want = 148LL * 3 * 4;
    int64_t maxn = 0;
    for (int s = 0; s < S; ++s) maxn = context_lens_host[s] > maxn ? context_lens_host[s] : maxn;
    auto items = [&](int64_t P) {
        int64_t it = 0;
        for (int s = 0; s < S; ++s) it += (context_lens_host[s] + P - 1) / P;
        return it * Hkv;
    };
    if (maxn == 0 || items(maxn) >= want) { *partition = 0; return PA_OK; }
    int64_t best = 256;
    for (int64_t P = 256; P < maxn; P *= 2)
        if (items(P) >= want) best = P;
    best = (best + bs - 1) / bs * bs;
    *partition = best >= maxn ? 0 : (int)best;
    return PA_OK;
}

extern "C" pa_status pa_decode_partition_group(int S, int Hq, int Hkv, int D, int bs,
                                               pa_dtype q_dt, pa_dtype cache_dt, int max_ctx,
                                               int partition, int num_sms, int* group) {
    clear_error();
    if (!group) return fail(PA_ERR_INVALID_ARG, "group is NULL");
    if (partition < 0) return fail(PA_ERR_INVALID_ARG, "partition must be >= 0 (no balanced grid)");
    pa_status chk = check_decode_shape(q_dt, cache_dt, S, Hq, Hkv, D, bs, max_ctx, partition);
    if (chk) return chk;
    const int G = Hq / Hkv;
    const int sel = g_select.load();
    const bool use_mma = !(sel & 1) && D <= 128 && cache_dt != PA_F32;
    const int64_t max_parts = partition > 0 ? parts_for(max_ctx, partition) : 1;
    const bool pair = bs == 8 && partition % 16 == 0;
    const int hg = decode_heads_per_cta(use_mma, pair ? 16 : bs, D, cache_dt, Hkv, sel) ? 4 : 1;
    *group = 1;
    if (use_mma && max_parts > 1)
        *group = (sel & 8) ? 3
                           : plan_part_group((int64_t)S * Hkv / hg, max_parts,
                                             (int64_t)partition * D * elem_size(cache_dt) * 2 * hg,
                                             num_sms > 0 ? num_sms : sm_count(), hg);
    return PA_OK;
}

extern "C" pa_status pa_decode_select(int mode) {
    clear_error();
    if (mode < 0 || mode > 127) return fail(PA_ERR_INVALID_ARG, "mode must be in [0, 127]");
    g_select.store(mode);
    return PA_OK;
}

int pa::decode_select_mode() { return g_select.load(); }

// pa_decode, plus the shared-prefix decode's two switches: the first
// `prefix_parts` partitions of sequences whose table starts with row 0's
// blocks were written by the prefix kernel, and every record goes through the
// workspace (force_ws) so the merge sees them all.
pa_status pa::decode_impl(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                          const void* value_cache, pa_dtype cache_dt, const int32_t* block_tables,
                          int MB, const int32_t* context_lens, int S, int Hq, int Hkv, int D,
                          int bs, int64_t NB, int max_ctx, float scale, float k_scale,
                          float v_scale, int partition, void* workspace, size_t workspace_bytes,
                          pa_stream_t stream, int prefix_parts, int force_ws,
                          int fuse_prefix_blocks) {
    pa_status chk = check_decode_shape(q_dt, cache_dt, S, Hq, Hkv, D, bs, max_ctx, partition);
    if (chk) return chk;
    if (MB < 0 || NB <= 0) return fail(PA_ERR_INVALID_ARG, "negative or zero size");
    const bool balanced = partition == PA_PARTITION_BALANCED;
    if (NB > 0x7fffffffLL) return fail(PA_ERR_INVALID_ARG, "NB exceeds int32 block ids");
    if (!(std::isfinite(scale)) || !(std::isfinite(k_scale) && k_scale > 0) ||
        !(std::isfinite(v_scale) && v_scale > 0))
        return fail(PA_ERR_INVALID_ARG, "scales must be finite (k_scale, v_scale > 0)");
    if (cache_dt != PA_FP8_E4M3 && (k_scale != 1.f || v_scale != 1.f))
        return fail(PA_ERR_INVALID_ARG, "k_scale / v_scale apply to fp8 caches only");
    const int G = Hq / Hkv;
    if (S == 0) return PA_OK;
    if (S > 65535 || (int64_t)Hkv * G > 65535) return fail(PA_ERR_UNSUPPORTED, "grid too large");
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens)
        return fail(PA_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned16(key_cache) || !aligned16(value_cache) || !aligned16(q) || !aligned16(out))
        return fail(PA_ERR_INVALID_ARG, "caches, q and out must be 16-byte aligned");
    if (MB == 0 && max_ctx > 0) return fail(PA_ERR_INVALID_ARG, "MB == 0 with max_ctx > 0");

    // shared-prefix decode: records up to partition prefix_parts exist even
    // when max_ctx ends inside the prefix (irregular sequences write them)
    const bool fuse = fuse_prefix_blocks > 0;
    const int64_t max_parts = balanced ? 1
                              : fuse ? prefix_parts            // the prefix records only
                              : prefix_parts > 0
                                  ? std::max<int64_t>(parts_for(max_ctx, partition), prefix_parts + 1)
                                  : parts_for(max_ctx, partition);
    if (max_parts > 65535 || (int64_t)Hkv * G > 65535)
        return fail(PA_ERR_UNSUPPORTED, "too many partitions or heads for the grid");
    // the suffix pass merges its warps' states and the prefix records with
    // weights kept behind the warp-merge area in its stage memory
    if (fuse && 4 * (4 * 16 * (D + 2) + (int64_t)G * (4 + prefix_parts + 2)) > 48 * 1024)
        return fail(PA_ERR_UNSUPPORTED, "shared prefix of %d partitions is too long", prefix_parts);
    const int sel = g_select.load();
    const bool use_mma = !(sel & 1) && D <= 128 && cache_dt != PA_F32;
    const int gc_simt = G < (D == 256 ? 2 : 4) ? G : (D == 256 ? 2 : 4);
    const int gc = use_mma ? G : gc_simt;
    const int chunks = use_mma ? 1 : G / gc_simt;
    const int num_sms = sm_count();
    // shared-prefix decode with whole suffixes: one CTA per (sequence, kv
    // head) item, or with bit 16 a persistent grid that streams the items back
    // to back, each CTA a run of whole items of about equal work
    const bool items = fuse && (sel & 16);
    // 8-token blocks go two to a stage (16 tokens) in the partition kernel,
    // where partitions are whole stages
    const bool pair = bs == 8 && !balanced && !fuse && prefix_parts == 0 && !force_ws &&
                      partition % 16 == 0;
    const int stage_tokens = pair ? 16 : bs;
    // four neighbouring kv heads per CTA (one per consumer warp), read by one
    // tensor-map copy per block and segment, where a stage of the four heads'
    // K and V is at most 32 KB (two stages in flight at three CTAs per SM);
    // one head per CTA with bit 32, the CUDA-core consumer, the balanced grid
    // and the shared-prefix suffix passes (short suffixes measured slower in
    // groups: four times fewer CTAs to hide their latency)
    const int hg = decode_heads_per_cta(use_mma, stage_tokens, D, cache_dt, Hkv, sel) &&
                           !balanced && !items && !force_ws && prefix_parts == 0
                       ? 4
                       : 1;
    int part_group = 1;
    if (use_mma && !balanced && !fuse && prefix_parts == 0 && !force_ws && max_parts > 1)
        part_group = (sel & 8) ? 3
                               : plan_part_group((int64_t)S * Hkv * chunks / hg, max_parts,
                                                 (int64_t)partition * D * elem_size(cache_dt) * 2 * hg,
                                                 num_sms, hg);
    const int64_t grid_parts = fuse ? 1
                               : prefix_parts > 0 ? max_parts - prefix_parts
                                                  : (max_parts + part_group - 1) / part_group;
    size_t need = 0;
    if (balanced) need = balanced_bytes(S, Hq, D, gc);
    else if (force_ws || fuse) need = (size_t)S * Hq * max_parts * (sizeof(float) * 2 + sizeof(float) * D);
    else pa_decode_workspace_size(S, Hq, D, max_ctx, partition, &need);
    if (force_ws && balanced) return fail(PA_ERR_INVALID_ARG, "the balanced grid has no prefix mode");
    if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
        return fail(PA_ERR_INVALID_ARG, "workspace needs %zu bytes, 16-byte aligned (got %zu)",
                    need, workspace_bytes);

    dec::Launch L{};
    pa_status st = hg > 1 ? make_cache_map_heads(&L.tmk, key_cache, cache_dt, NB, bs, Hkv, D, hg)
                          : make_cache_map(&L.tmk, key_cache, cache_dt, NB, bs, Hkv, D);
    if (st) return st;
    st = hg > 1 ? make_cache_map_heads(&L.tmv, value_cache, cache_dt, NB, bs, Hkv, D, hg)
                : make_cache_map(&L.tmv, value_cache, cache_dt, NB, bs, Hkv, D);
    if (st) return st;
    unsigned int* err = device_error_word();
    if (!err) return PA_ERR_CUDA;

    dec::Params& p = L.p;
    p.out = out;
    p.q = q;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.err = err;
    p.S = S;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.MB = MB;
    p.max_parts = (int)max_parts;
    p.part_blocks = !fuse && (max_parts > 1 || force_ws) ? partition / stage_tokens : 0;
    p.part_tokens = !fuse && (max_parts > 1 || force_ws) ? partition : 0;
    p.prefix_parts = prefix_parts;
    p.force_ws = force_ws ? 1 : 0;
    p.fuse_prefix_blocks = fuse_prefix_blocks;
    p.part_group = part_group;
    // one CTA per suffix: room for the prefix records behind the stage
    // barriers, fetched while the suffix streams (records and their offsets
    // 16-byte aligned: an even record count per head, or an even number of
    // heads per CTA starting at an even head)
    p.rec_smem = 0;
    if (fuse && !items && (max_parts % 2 == 0 || (gc % 2 == 0 && G % 2 == 0))) {
        const size_t rb = 16 + (size_t)gc * hg * max_parts * ((size_t)D * 4 + 8);
        if (rb <= 12 * 1024) p.rec_smem = (int)rb;
    }
    p.max_ctx = max_ctx;
    p.evict_first = (sel & 2) ? 1 : 0;
    p.heads_fastest = (sel & 4) ? 1 : 0;
    p.NB = NB;
    p.qk_scale = (float)((double)scale * (double)k_scale * 1.4426950408889634);
    p.v_scale = v_scale;
    p.bs = bs;
    p.gc = gc;
    p.balanced = balanced || items ? 1 : 0;
    p.whole_items = items ? 1 : 0;
    if (balanced) {
        const size_t items = (size_t)S * (Hq / gc);
        const size_t rows = (items + dec::kMaxBalancedCtas) * gc;
        char* w = static_cast<char*>(workspace);
        p.ws_item = reinterpret_cast<int2*>(w);
        p.ws_rows = (int64_t)rows;
        p.ws_ml = reinterpret_cast<float2*>(w + align16(items * sizeof(int2)));
        p.ws_o = reinterpret_cast<float*>(w + align16(items * sizeof(int2)) +
                                          align16(rows * sizeof(float2)));
    } else if (max_parts > 1 || force_ws || fuse) {
        p.ws_ml = static_cast<float2*>(workspace);
        p.ws_o = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          sizeof(float2) * (size_t)S * Hq * max_parts);
    }

    L.bs = bs;
    L.pair = pair;
    L.hg = hg;
    L.D = D;
    L.mma = use_mma;
    L.mrows = G <= 8 ? 8 : 16;
    L.gc = gc_simt;
    L.balanced = balanced || items;
    L.G = G;
    L.num_sms = num_sms;
    const unsigned head_ctas = (unsigned)(Hkv * chunks / hg);
    L.grid = p.heads_fastest ? dim3(head_ctas, (unsigned)grid_parts, (unsigned)S)
                             : dim3((unsigned)grid_parts, head_ctas, (unsigned)S);
    L.stream = reinterpret_cast<cudaStream_t>(stream);

    cudaError_t e;
    switch (cache_dt) {
    case PA_F32: e = dec::launch_f32(L); break;
    case PA_F16: e = dec::launch_f16(L); break;
    case PA_BF16: e = dec::launch_bf16(L); break;
    default: e = q_dt == PA_F16 ? dec::launch_fp8_q_f16(L) : dec::launch_fp8_q_bf16(L); break;
    }
    if (e == cudaErrorNotSupported) return fail(PA_ERR_UNSUPPORTED, "no kernel for this shape");
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    if (!fuse && (max_parts > 1 || balanced || force_ws)) {
        e = launch_merge(p, q_dt, D, Hq, S, L.stream);
        if (e != cudaSuccess) return cuda_fail(e, "split-K merge launch");
    }
    return PA_OK;
}

extern "C" pa_status pa_decode(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                               const void* value_cache, pa_dtype cache_dt,
                               const int32_t* block_tables, int MB, const int32_t* context_lens,
                               int S, int Hq, int Hkv, int D, int bs, int64_t NB, int max_ctx,
                               float scale, float k_scale, float v_scale, int partition,
                               void* workspace, size_t workspace_bytes, pa_stream_t stream) {
    PA_NVTX_RANGE("pa_decode");
    clear_error();
    return decode_impl(out, q, q_dt, key_cache, value_cache, cache_dt, block_tables, MB,
                       context_lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale, k_scale, v_scale,
                       partition, workspace, workspace_bytes, stream, 0, 0, 0);
}
