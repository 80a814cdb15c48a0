/*
 * pa.h -- C ABI of the paged decode library (libpa_b200.so, sm_100a).
 *
 * The library implements single-token decode attention over a KV cache kept
 * in fixed-size physical blocks ("PagedAttention 机制" §5.3.1-§5.3.4;
 * "01. PagedAttention 详解" §3-§6), together with the cache append, the
 * copy-on-write block copy and a host-side refcounted block pool.
 *
 * Conventions for every function:
 *   - Returns a pa_status; PA_OK is 0.  No exception crosses this boundary.
 *     pa_last_error() gives a message for the last failure on the calling
 *     thread.
 *   - Device pointers are plain CUDA device addresses; the CALLER owns and
 *     allocates all device memory (caches, q, out, tables, workspace).  The
 *     library allocates no device memory.
 *   - Device work is enqueued asynchronously on the caller's stream
 *     (pa_stream_t is cudaStream_t; NULL is the legacy default stream).
 *     Argument checks are done on the host before anything is enqueued; a
 *     failed check enqueues nothing.  A launch failure returns PA_ERR_CUDA.
 *   - Values that live in device memory (block ids, slots) cannot be checked
 *     on the host without a synchronisation.  The kernels check them, skip the
 *     offending access (a TMA load outside the cache reads zeros; a store is
 *     dropped) and set a sticky bit readable with pa_device_status().  No
 *     kernel here traps, asserts, or waits without a bound.
 *
 * Layouts ("01. PagedAttention 详解" §3, the cache shape of its
 * FlashAttention backend), all row-major:
 *   key_cache, value_cache : [NB, bs, Hkv, D]     physical blocks
 *   q, out                 : [S, Hq, D]
 *   block_tables           : [S, MB] int32         physical block ids
 *   context_lens           : [S] int32             tokens to attend, >= 0
 *   slot_mapping           : [T] int64             block * bs + offset, < 0 skips
 *   key, value (append)    : [T, Hkv, D]
 * where S = sequences, Hq / Hkv = query / kv heads (Hq % Hkv == 0, query head
 * h reads kv head h / (Hq / Hkv)), D = head dim, bs = block size, NB = number
 * of physical blocks, MB = table width.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* pa_stream_t; /* same type as cudaStream_t */

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* a size, pointer, dtype or value is not acceptable */
    PA_ERR_UNSUPPORTED = 2,   /* valid, but no kernel is built for this shape/dtype */
    PA_ERR_OUT_OF_BLOCKS = 3, /* the pool has no free block (state unchanged) */
    PA_ERR_REFCOUNT = 4,      /* free of a free block, sharing a free block */
    PA_ERR_BAD_INDEX = 5,     /* unknown sequence / block id (host side) */
    PA_ERR_CUDA = 6           /* a CUDA runtime call failed */
} pa_status;

typedef enum {
    PA_F32 = 0,
    PA_F16 = 1,
    PA_BF16 = 2,
    PA_FP8_E4M3 = 3 /* OCP E4M3 "FN": bias 7, max 448, no inf, S.1111.111 = NaN */
} pa_dtype;

/* Device-side error bits (sticky until read with clear != 0). */
enum {
    PA_DEV_BAD_SLOT = 1,      /* pa_reshape_and_cache: slot >= NB * bs, token skipped */
    PA_DEV_BAD_BLOCK = 2,     /* pa_decode: table entry outside [0, NB) (read as zeros) */
    PA_DEV_WAIT_TIMEOUT = 4,  /* a pipeline wait gave up after its bound; output invalid */
    PA_DEV_BAD_CONTEXT = 8,   /* pa_decode: context_lens[s] < 0, > max_ctx or > MB * bs (clamped) */
    PA_DEV_BAD_PIECES = 16    /* pa_decode merge: inconsistent split records (rows left unwritten) */
};
/* Bits 16-23 of the device word, when PA_DEV_WAIT_TIMEOUT is set: which wait
 * gave up last (diagnostics; decode: 1 stage-free, 2 stage-full,
 * 3 descriptor-free, 4 descriptor-ready, 5 states-published, 6 merge-done,
 * 19 prefix-records;
 * prefill: 7 q-tile, 8 k-tile-full, 9 v-tile-full, 10 k-tile-free,
 * 11 v-tile-free, 12 scores-ready, 13 probabilities-ready, 14 p.v-done,
 * 15 output-ready, 16 tensor-core drain, 17 load drain, 18 exponential turn). */

/* Message for the last failing call on this thread ("" if none). */
const char* pa_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int pa_version(void);

/*
 * Kernels this library has enqueued since the process loaded it, over every
 * device and stream (a launch that failed is not counted).  The difference
 * between two reads is the number of the library's kernels a stretch of host
 * code launched.  No citation: bookkeeping of this library, not of the method.
 */
uint64_t pa_launch_count(void);

/*
 * Read (and with clear != 0, reset) the sticky device error bits of the
 * current device.  Synchronises `stream` first so the bits cover all work
 * enqueued on it.
 */
pa_status pa_device_status(unsigned int* bits, int clear, pa_stream_t stream);

/*
 * Cache append -- "01. PagedAttention 详解" §4, decode step 2 (write the new
 * token's k, v into the next slot of the last block) and prefill step 2 (write
 * N tokens' K, V through the block table).
 *
 * For every t < T with slot = slot_mapping[t] >= 0, b = slot / bs,
 * o = slot % bs:  key_cache[b, o, h, :] = cvt(key[t, h, :]) for all h, and the
 * same for value.  cvt is a byte copy when in_dt == cache_dt.  With
 * cache_dt == PA_FP8_E4M3 (intelliparadigm PagedAttention article §4.3,
 * kv_cache_dtype "fp8"), cvt(x) rounds x / k_scale (binary32 division) to the
 * nearest E4M3 value, ties to even, saturating at +-448; in_dt is then
 * PA_F32, PA_F16 or PA_BF16.  Other dtype pairs: PA_ERR_UNSUPPORTED.
 * k_scale and v_scale must be finite and > 0, and 1.0 unless the cache is fp8.
 *
 * key, value: device [T, Hkv, D] in_dt.  slot_mapping: device int64 [T].
 * A slot >= NB * bs is skipped and sets PA_DEV_BAD_SLOT.  Two tokens with the
 * same slot: one of them wins (unspecified which).  T == 0 is a no-op.
 * D * element size must be a multiple of 16 bytes; pointers 16-byte aligned.
 */
pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype in_dt,
                               void* key_cache, void* value_cache, pa_dtype cache_dt,
                               const int64_t* slot_mapping, int T, int Hkv, int D, int bs,
                               int64_t NB, float k_scale, float v_scale, pa_stream_t stream);

/*
 * Copy-on-write block copy -- intelliparadigm PagedAttention article §3.3
 * (maybe_copy_block: allocate, copy_block, drop the old reference) and
 * "PagedAttention 机制" §5.3.2 (copy only when a shared block is written).
 *
 * For each pair i: key_cache block pairs[2i+1] = key_cache block pairs[2i]
 * (all block_bytes of it), and the same for value_cache.  block_bytes is
 * bs * Hkv * D * element size and must be a multiple of 16.
 * pairs: HOST int32 [n, 2] (src, dst) -- the pool decides copies on the host,
 * and the list travels in the kernel's parameters, so no device buffer is
 * needed.  Rejected on the host (PA_ERR_INVALID_ARG): an id outside [0, NB), a
 * destination that repeats, a destination that is also a source.
 * n == 0 is a no-op.
 */
pa_status pa_copy_blocks(void* key_cache, void* value_cache, size_t block_bytes, int64_t NB,
                         const int32_t* pairs, int n, pa_stream_t stream);

/* partition value selecting the persistent work-balanced decode (see pa_decode) */
#define PA_PARTITION_BALANCED (-1)

/*
 * Bytes of split-K workspace pa_decode needs for these sizes: 0 when
 * partition == 0 or max_ctx <= partition; for fixed partitions, per
 * (s, query head, partition) a running max m, a sum l and an unnormalised
 * o[D] in fp32; for PA_PARTITION_BALANCED, an upper bound covering every
 * kernel choice (per-item piece bounds plus one partial per piece).
 */
pa_status pa_decode_workspace_size(int S, int Hq, int D, int max_ctx, int partition,
                                   size_t* bytes);

/*
 * Split size pa_decode would pick for this batch to fill the GPU: a multiple
 * of bs, or 0 for a single pass.  Host-only heuristic, no device access.
 */
pa_status pa_decode_suggest_partition(int S, int Hkv, int bs, const int32_t* context_lens_host,
                                      int* partition);

/*
 * Paged decode attention -- "PagedAttention 机制" §5.3.4 (paged_attention:
 * logical token i is key_cache[block_tables[i // bs], i % bs]);
 * intelliparadigm PagedAttention article §2.3 (q.K per block, softmax
 * normalised over all blocks, weighted sum of V); "01. PagedAttention 详解" §4
 * (per-block partial results accumulated; v2 splits long sequences, split-K).
 *
 * For every s < S and query head h, g = h / (Hq / Hkv), n = context_lens[s]:
 *   k_i = deq(key_cache[block_tables[s, i / bs], i % bs, g, :]),  i < n
 *   z_i = scale * <q[s, h, :], k_i>
 *   out[s, h, :] = sum_i softmax(z)_i * deq(value_cache[..same slot.., g, :])
 * deq(x) = x * k_scale (keys) or x * v_scale (values) for fp8, x otherwise.
 * Accumulation is fp32; out is rounded to nearest-even in q_dt.  n == 0 gives
 * a zero row.  Table entries at or past ceil(n / bs) and cache slots at or
 * past n are never read.
 *
 * dtypes: cache_dt == q_dt for F32 / F16 / BF16; cache_dt == PA_FP8_E4M3 with
 * q_dt F16 or BF16.  bs in {8, 16, 32}; D in {64, 128, 256} with D * element
 * size of the cache in {128, 256, 512} bytes; Hq / Hkv in {1, 2, 4, 8, 16}.
 * Base pointers 16-byte aligned (TMA requirement).
 *
 * partition: 0 = one pass per (sequence, kv head); a positive multiple of bs
 * = tokens per split-K partition: sequences longer than one partition are
 * split, each partition writes (m, l, o) into `workspace` and a second kernel
 * on the same stream merges them; PA_PARTITION_BALANCED = a persistent grid
 * sized to the GPU whose CTAs take equal contiguous shares of all blocks of
 * all (sequence, kv head) items (items cut at share boundaries are merged
 * the same way).  `workspace`: device, >= pa_decode_workspace_size() bytes,
 * 16-byte aligned, no initialisation needed.  max_ctx must be >= every
 * context_lens[s] (it sizes the grid and the workspace).
 */
pa_status pa_decode(void* out, const void* q, pa_dtype q_dt,
                    const void* key_cache, const void* value_cache, pa_dtype cache_dt,
                    const int32_t* block_tables, int MB, const int32_t* context_lens,
                    int S, int Hq, int Hkv, int D, int bs, int64_t NB, int max_ctx,
                    float scale, float k_scale, float v_scale, int partition,
                    void* workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode without a caller-provided workspace.  (The pages have no
 * counterpart of this entry point: it exists for callers of this library.)
 *
 * For callers that cannot allocate device memory for the split-K partials:
 * a serving runtime that hands all device memory to its KV cache at start-up
 * and owns the only allocator, a plugin inside a framework that exposes no
 * allocation hook, or a step loop that must not call cudaMalloc / cudaFree
 * (cudaFree waits for the whole device) while it runs.  Same arguments and
 * result as pa_decode, minus the workspace: the partials live in a fixed
 * device array of PA_DECODE_NOALLOC_SCRATCH_BYTES inside the library, which
 * every GPU that loads the library holds until the process exits.  This
 * function allocates nothing.
 *
 * Limits: if pa_decode_workspace_size() for these sizes exceeds the array,
 * the call fails with PA_ERR_INVALID_ARG before enqueuing anything (choose a
 * larger partition, or use pa_decode).  All calls share the one array, so
 * calls whose device work may overlap (different streams or host threads)
 * race on it: the caller must order them.  Nothing in the array needs to
 * start at zero; a call reads only partials it wrote itself.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it with the
 * device's context; make that first call before any stream capture.  After a
 * cudaDeviceReset the device has a new context, and the next call looks the
 * address up again (again: outside any capture).
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20) /* 32 MiB */
pa_status pa_decode_noalloc(void* out, const void* q, pa_dtype q_dt,
                            const void* key_cache, const void* value_cache, pa_dtype cache_dt,
                            const int32_t* block_tables, int MB, const int32_t* context_lens,
                            int S, int Hq, int Hkv, int D, int bs, int64_t NB, int max_ctx,
                            float scale, float k_scale, float v_scale, int partition,
                            pa_stream_t stream);

/*
 * How many consecutive split-K partitions one pa_decode CTA streams for this
 * shape (the grouped path of bit 8 below; each partition still writes its own
 * record, so the result does not depend on it).  Plain split-K (partition >
 * 0) with the tensor-core consumer only; num_sms <= 0 means the current
 * device's SM count (148 without a device).  It is the planned value: the
 * launch falls back to 1 where the group's merge area would cost a resident
 * CTA per SM (fp8 tiles, 16-head groups).  *group >= 1 on success.
 * The shape and dtype rules are pa_decode's (same return codes for a shape
 * pa_decode would refuse); partition must be >= 0.
 */
pa_status pa_decode_partition_group(int S, int Hq, int Hkv, int D, int bs, pa_dtype q_dt,
                                    pa_dtype cache_dt, int max_ctx, int partition, int num_sms,
                                    int* group);

/*
 * Kernel selection and tuning for pa_decode and pa_prefill (process-wide; for tests and
 * tuning), a bit mask:
 *   1: CUDA-core consumer everywhere (otherwise f16 / bf16 / fp8 caches with
 *      D <= 128 use the tensor-core consumer, multi-head attention included:
 *      its one query row per kv head fills one of the tile's eight);
 *   2: stream K/V with an L2 evict-first hint;
 *   4: partition-major grid (the kv heads of one partition are neighbouring
 *      CTAs, so the interleaved heads of a block are read at about the same
 *      time); otherwise kv-head-major;
 *   8: with split-K partitions, one CTA streams three consecutive partitions
 *      whenever there are several (the grouped path at any size; without
 *      this bit it is taken for partitions under 512 KB of K/V per kv head,
 *      with the count per CTA that minimises full waves of resident CTAs
 *      times each CTA's bytes plus its start-up).
 *      Each partition still gets its own record, so the result is the same.
 *      Tensor-core consumer only, and only where the CTA's extra merge area
 *      costs no resident CTA per SM.
 *  16: pa_decode_shared_prefix with suffixes of at most 4096 tokens: a
 *      persistent grid in groups of one CTA per kv head, each group streaming
 *      a run of whole sequences' suffixes of about equal total length without
 *      draining its pipeline, instead of the default one CTA per (sequence,
 *      kv head) suffix.
 *  32: one kv head per CTA everywhere.  Otherwise, with the tensor-core
 *      consumer and Hkv a multiple of 4, a CTA of the partition kernel serves
 *      four neighbouring kv heads (one per consumer warp) and reads each
 *      block's rows of all four with one tensor-map copy per 128-byte
 *      segment (grouped partitions included: each warp then closes its
 *      head's partition records alone; not with the balanced grid or the
 *      shared-prefix decode's suffix passes).
 *  64: pa_prefill with D = 128 (outside the shared-prefix decode) runs the
 *      two query tiles of a pair on a cluster of two CTAs whose tensor-core
 *      instructions span both SMs (cta_group::2: each SM loads half of every
 *      K and V tile and keeps two score buffers, so the scores of the next key
 *      tile are computed while the softmax works on this one) instead of one
 *      CTA per pair.  Same results; measured about 6 % slower.
 * Default 4; a mode outside [0, 127] is refused (PA_ERR_INVALID_ARG).
 * Every setting computes the same function.
 */
pa_status pa_decode_select(int mode);

/*
 * Shared-prefix ("cascade") decode -- "01. PagedAttention 详解" §6 and summary
 * (requests share the blocks of a common prefix by reference) and
 * "PagedAttention 机制" §5.3.2.  Computes exactly what pa_decode computes (up
 * to rounding order), for a batch whose block tables all start with the same
 * prefix_tokens / bs physical blocks (those of row 0): the prefix is attended
 * once, by a tensor-core pass with every sequence's queries as rows, and each
 * sequence's private suffix by the decode kernel; the split-K merge combines
 * them.  A sequence whose table does not start with row 0's prefix blocks, or
 * that holds fewer than prefix_tokens tokens, is still computed correctly
 * (it reads its own prefix blocks).
 *
 * Arguments are pa_decode's (same layouts, ownership, errors) except:
 *   prefix_tokens  host int, a positive multiple of bs, <= MB * bs;
 *   workspace      device scratch of pa_decode_shared_prefix_workspace_size()
 *                  bytes, 16-byte aligned (no initialisation needed).
 * Supported: q f16 or bf16 with a cache of the same type or fp8-e4m3 (the
 * prefix is converted exactly to the q type inside the workspace), D in
 * {64, 128} (128 for fp8: a row is at least 128 bytes), Hq / Hkv in
 * {1, 2, 4, 8, 16}, bs in {8, 16, 32}; scale > 0.
 * With max_ctx < prefix_tokens it is a plain pa_decode.
 */
pa_status pa_decode_shared_prefix_workspace_size(int S, int Hq, int Hkv, int D, int bs,
                                                 int max_ctx, int prefix_tokens,
                                                 pa_dtype cache_dt, size_t* bytes);
pa_status pa_decode_shared_prefix(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                                  const void* value_cache, pa_dtype cache_dt,
                                  const int32_t* block_tables, int MB,
                                  const int32_t* context_lens, int S, int Hq, int Hkv, int D,
                                  int bs, int64_t NB, int max_ctx, float scale, float k_scale,
                                  float v_scale, int prefix_tokens, void* workspace,
                                  size_t workspace_bytes, pa_stream_t stream);

/*
 * Prefill / chunked-prefill attention over the paged cache -- "01. PagedAttention
 * 详解" §4, prefill: the N new tokens' K and V are first written through the
 * block table (pa_reshape_and_cache with their slots), then attention runs
 * over the cache.  Sequence s holds n_s = context_lens[s] tokens in the cache,
 * of which the last L_s = query_start[s+1] - query_start[s] are this call's new
 * tokens, rows query_start[s] .. query_start[s+1]-1 of q.  New token i sits at
 * position p = n_s - L_s + i and attends causally to the keys at 0..p:
 *
 *   out[row, h, :] = softmax(scale * K_s[0..p] q[row, h, :]) V_s[0..p]
 *
 * with K_s, V_s gathered through block_tables exactly as in pa_decode (kv head
 * h / (Hq / Hkv)).  L_s = n_s is a prefill from an empty cache, L_s < n_s a
 * chunk of a chunked prefill (or a prefix-cache hit), L_s = 1 a decode step.
 *
 * Arguments (device pointers unless stated):
 *   out, q       [T, Hq, D] of q_dt, T = query_start[S]; rows of one sequence
 *                are contiguous.  16-byte aligned.
 *   key_cache, value_cache  [NB, bs, Hkv, D] of cache_dt; cache_dt must equal
 *                q_dt (PA_F16 or PA_BF16: the tensor cores take both operands
 *                in one type); other dtypes return PA_ERR_UNSUPPORTED.
 *   block_tables [S, MB] int32; context_lens [S] int32;
 *   query_start  [S+1] int32, non-decreasing, query_start[0] = 0.
 *   max_query_len  host int >= every L_s (sizes the grid).
 *   scale        host float, finite and > 0.
 *   D in {64, 128}; Hq / Hkv in {1, 2, 4, 8, 16}; bs in {8, 16, 32}.
 * Work runs asynchronously on `stream` with no allocation and no workspace.
 * Host checks return PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED before anything is
 * enqueued.  Device-side, a table entry outside [0, NB) sets PA_DEV_BAD_BLOCK
 * (its keys are read as whatever the tile held: the rows that need them are
 * invalid); L_s > n_s, L_s > max_query_len or n_s > MB * bs sets
 * PA_DEV_BAD_CONTEXT and the sequence's rows are left unwritten.
 */
pa_status pa_prefill(void* out, const void* q, pa_dtype q_dt, const void* key_cache,
                     const void* value_cache, pa_dtype cache_dt, const int32_t* block_tables,
                     int MB, const int32_t* context_lens, const int32_t* query_start, int S,
                     int T, int Hq, int Hkv, int D, int bs, int64_t NB, int max_query_len,
                     float scale, pa_stream_t stream);

/* ------------------------------------------------------------------------
 * Host block pool -- "PagedAttention 机制" §5.3.4 (BlockAllocator: free list,
 * per-block reference count, allocate / free / incr_ref, out-of-memory when
 * empty) with the FIFO free queue of "01. PagedAttention 详解" self-check 3
 * (get_new_blocks takes from the head, free_blocks returns a block to the
 * tail when its count reaches 0), per-sequence block tables ("PagedAttention
 * 机制" §5.3.2), sharing by reference counts ("01. PagedAttention 详解" §6
 * and its summary: prefix sharing, beam search and parallel sampling) and
 * copy-on-write (intelliparadigm
 * PagedAttention article §3.3).
 *
 * Not thread-safe: one scheduler thread owns a pool.  No device access.
 * Sequence ids are int64 handles returned by the pool.
 * ------------------------------------------------------------------------ */
typedef struct pa_pool pa_pool;

typedef struct {
    int64_t num_blocks;
    int64_t free_blocks;
    int64_t used_blocks;    /* reference count > 0 */
    int64_t shared_blocks;  /* reference count > 1 */
    int64_t cow_copies;     /* copies requested by pa_pool_seq_append so far */
    int64_t num_seqs;
    int64_t cached_blocks;  /* blocks holding a registered content hash */
    int64_t cache_hits;     /* prefix-cache hits so far */
} pa_pool_stats_t;

pa_status pa_pool_create(int64_t NB, int bs, pa_pool** out);
void pa_pool_destroy(pa_pool* pool);

/* Take the head of the free queue; its count becomes 1. */
pa_status pa_pool_alloc(pa_pool* pool, int32_t* block);
/* Drop one reference; at 0 the block goes to the tail of the free queue. */
pa_status pa_pool_free(pa_pool* pool, int32_t block);
/* Add a reference to a block in use (PA_ERR_REFCOUNT if it is free). */
pa_status pa_pool_incr_ref(pa_pool* pool, int32_t block);
/* Reference count of a block (-1 if the id is out of range). */
int pa_pool_ref(const pa_pool* pool, int32_t block);

/* New empty sequence. */
pa_status pa_pool_seq_new(pa_pool* pool, int64_t* seq);
/* New sequence sharing all of parent's blocks (one more reference each).
 * PA_ERR_REFCOUNT (and no change) if one of them was freed behind the pool's back. */
pa_status pa_pool_seq_fork(pa_pool* pool, int64_t parent, int64_t* child);
/*
 * An EMPTY sequence takes a reference on n existing blocks holding its first
 * num_tokens tokens (a shared prefix); n must equal ceil(num_tokens / bs).
 */
pa_status pa_pool_seq_share_prefix(pa_pool* pool, int64_t seq, const int32_t* blocks, int n,
                                   int64_t num_tokens);
/*
 * Make room for one more token of `seq` and return its slot
 * (block * bs + offset).  A new block is taken when the last one is full.  If
 * the last block is shared (count > 1) it is copied first: a fresh block is
 * taken, *cow_src / *cow_dst name the copy the caller must enqueue (with
 * pa_copy_blocks, before writing the slot), the old block loses one reference
 * and the table now points at the new one; otherwise both are -1.  On
 * PA_ERR_OUT_OF_BLOCKS nothing changes.
 */
pa_status pa_pool_seq_append(pa_pool* pool, int64_t seq, int64_t* slot, int32_t* cow_src,
                             int32_t* cow_dst);
/*
 * pa_pool_seq_append for each of n distinct sequences, in order, in one call
 * (one decode step of a batch).  slots[i] receives sequence i's slot;
 * cow_pairs receives the *n_cow (src, dst) copies to enqueue with
 * pa_copy_blocks before the append kernel (room for n pairs).  All or
 * nothing: an unknown or repeated sequence, or fewer free blocks than the
 * batch needs, returns an error and changes nothing.
 */
pa_status pa_pool_seq_append_batch(pa_pool* pool, const int64_t* seqs, int n, int64_t* slots,
                                   int32_t* cow_pairs, int* n_cow);
/* Drop the sequence's reference on each of its blocks, in table order.  All
 * or nothing: PA_ERR_REFCOUNT (and no change) if a block holds fewer
 * references than the sequence does. */
pa_status pa_pool_seq_free(pa_pool* pool, int64_t seq);
/* Tokens held by a sequence (-1 if unknown). */
int64_t pa_pool_seq_len(const pa_pool* pool, int64_t seq);

/*
 * Pack the tables of `seqs` into one host buffer for one host-to-device copy
 * per step ("01. PagedAttention 详解" §10: all active tables go to the GPU as
 * one tensor, not one small copy per request).  tables_host: [S, MB] int32,
 * entries past a sequence's blocks are -1; ctx_lens_host: [S] int32.
 * PA_ERR_INVALID_ARG if a sequence holds more than MB blocks.
 */
pa_status pa_pool_build_block_tables(const pa_pool* pool, const int64_t* seqs, int S, int MB,
                                     int32_t* tables_host, int32_t* ctx_lens_host);

pa_status pa_pool_stats(const pa_pool* pool, pa_pool_stats_t* stats);

/*
 * One decode step's host work in one call: pa_pool_seq_append_batch on
 * `seqs`, then pa_pool_build_block_tables of the same sequences into
 * tables_host [n, MB] / ctx_lens_host [n] (the lengths include the token just
 * appended).  All or nothing: an unknown or repeated sequence, a table that
 * would need more than MB entries, or too few free blocks returns an error
 * and changes nothing.
 */
pa_status pa_pool_step(pa_pool* pool, const int64_t* seqs, int n, int MB, int64_t* slots,
                       int32_t* cow_pairs, int* n_cow, int32_t* tables_host,
                       int32_t* ctx_lens_host);

/* The physical blocks of a sequence, in table order (*n is set even when cap
 * is too small, which returns PA_ERR_INVALID_ARG). */
pa_status pa_pool_seq_blocks(const pa_pool* pool, int64_t seq, int32_t* blocks, int cap, int* n);

/*
 * Prefix cache -- "01. PagedAttention 详解" self-check 3 and summary: a
 * prefix-cache hit hands an already filled block to a new request by adding
 * a reference (_get_cached_block: ref_cnt++), and freed blocks are reused in
 * LRU order.  The caller names the content of a FULL block by a 64-bit hash
 * of its own choosing (e.g. of the token ids it holds and of the previous
 * block's hash).
 *
 * pa_pool_cache_block: remember that `block` (in use) holds content `hash`.
 *   *cached = 1 if it is now the block for that hash; 0 if another block
 *   already holds it.  A block whose count drops to 0 keeps its content and
 *   hash while it waits in the free queue; taking it from the queue head for
 *   a new allocation forgets the hash (eviction of the least recently freed).
 *   Appending into a block the sequence holds alone forgets its hash.
 * pa_pool_cache_lookup: *block = the block holding `hash` with one more
 *   reference taken (a freed one leaves the free queue with count 1), or -1.
 * pa_pool_seq_match_prefix: an EMPTY sequence takes the blocks of the longest
 *   run of leading hashes that hit, one reference each; *matched = that count
 *   and the sequence then holds matched * bs tokens.
 */
pa_status pa_pool_cache_block(pa_pool* pool, int32_t block, uint64_t hash, int* cached);
pa_status pa_pool_cache_lookup(pa_pool* pool, uint64_t hash, int32_t* block);
pa_status pa_pool_seq_match_prefix(pa_pool* pool, int64_t seq, const uint64_t* hashes, int n,
                                   int* matched);

/*
 * Sequence sharding over several GPUs (host only; the pages have no
 * counterpart: they describe one GPU).  Decode reads no other sequence's
 * blocks, so a batch splits by sequence with no exchange between devices;
 * each device then runs its own step over its own cache.  The plan balances
 * the K/V bytes each device streams, which are proportional to the context
 * lengths: sequences are taken longest first (ties: lower index first) and
 * each goes to the device with the fewest tokens so far (ties: lower device).
 *
 * context_lens_host: [S] lengths (>= 0).  device_of_seq_host: [S] out, the
 * device of each sequence.  tokens_per_device_host: [ndev] out (may be NULL).
 * S >= 0, ndev >= 1, else PA_ERR_INVALID_ARG.
 */
pa_status pa_plan_shards(const int32_t* context_lens_host, int S, int ndev,
                         int32_t* device_of_seq_host, int64_t* tokens_per_device_host);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
