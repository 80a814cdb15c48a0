"""Python binding of libpa_b200.so: paged decode attention on B200 (sm_100a).

Thin ctypes marshalling over the C ABI declared in include/pa.h -- every
function here has the name of the C entry point it calls, takes torch tensors
(device memory, owned by the caller) and passes their pointers, sizes and
dtypes through.  All computation happens in the library's CUDA kernels; there
is no fallback: if the shared library is missing or fails to load, every call
raises.

Build the library with ``python -m paged_kv_cache_338_b200.build`` (or
``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

__all__ = [
    "PaError", "lib", "pa_version", "pa_launch_count", "pa_last_error", "pa_device_status",
    "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_workspace_size",
    "pa_decode_suggest_partition", "pa_decode_partition_group", "pa_decode_select", "pa_decode_noalloc", "pa_prefill",
    "pa_decode_shared_prefix", "pa_decode_shared_prefix_workspace_size",
    "BlockPool", "pa_plan_shards",
    "PA_DEV_BAD_SLOT", "PA_DEV_BAD_BLOCK", "PA_DEV_WAIT_TIMEOUT", "PA_DEV_BAD_CONTEXT",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

# pa_status / pa_dtype / device error bits (include/pa.h)
STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED",
          3: "PA_ERR_OUT_OF_BLOCKS", 4: "PA_ERR_REFCOUNT", 5: "PA_ERR_BAD_INDEX",
          6: "PA_ERR_CUDA"}
PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
PA_DEV_BAD_SLOT, PA_DEV_BAD_BLOCK, PA_DEV_WAIT_TIMEOUT, PA_DEV_BAD_CONTEXT = 1, 2, 4, 8
PA_DEV_BAD_PIECES = 16

_TORCH_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16,
             torch.float8_e4m3fn: PA_FP8_E4M3, torch.uint8: PA_FP8_E4M3}


class PaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = STATUS.get(status, str(status))
        super().__init__(f"{self.status}: {msg}")


class _Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in
                ("num_blocks", "free_blocks", "used_blocks", "shared_blocks", "cow_copies",
                 "num_seqs", "cached_blocks", "cache_hits")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is not built (no CPU fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m paged_kv_cache_338_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I32, I64, F, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_int64,
                             ctypes.c_float, ctypes.c_size_t)
    sig = {
        "pa_last_error": ([], ctypes.c_char_p),
        "pa_version": ([], I),
        "pa_launch_count": ([], ctypes.c_uint64),
        "pa_device_status": ([ctypes.POINTER(ctypes.c_uint), I, P], I),
        "pa_reshape_and_cache": ([P, P, I, P, P, I, P, I, I, I, I, I64, F, F, P], I),
        "pa_copy_blocks": ([P, P, SZ, I64, P, I, P], I),
        "pa_decode_workspace_size": ([I, I, I, I, I, ctypes.POINTER(SZ)], I),
        "pa_decode_suggest_partition": ([I, I, I, P, ctypes.POINTER(I)], I),
        "pa_decode_partition_group": ([I, I, I, I, I, I, I, I, I, I, ctypes.POINTER(I)], I),
        "pa_decode_select": ([I], I),
        "pa_decode": ([P, P, I, P, P, I, P, I, P, I, I, I, I, I, I64, I, F, F, F, I, P, SZ, P], I),
        "pa_decode_noalloc": ([P, P, I, P, P, I, P, I, P, I, I, I, I, I, I64, I, F, F, F, I, P], I),
        "pa_prefill": ([P, P, I, P, P, I, P, I, P, P, I, I, I, I, I, I, I64, I, F, P], I),
        "pa_decode_shared_prefix_workspace_size": ([I, I, I, I, I, I, I, I, ctypes.POINTER(SZ)], I),
        "pa_decode_shared_prefix": ([P, P, I, P, P, I, P, I, P, I, I, I, I, I, I64, I, F, F, F, I,
                                     P, SZ, P], I),
        "pa_pool_create": ([I64, I, ctypes.POINTER(P)], I),
        "pa_pool_destroy": ([P], None),
        "pa_pool_alloc": ([P, ctypes.POINTER(I32)], I),
        "pa_pool_free": ([P, I32], I),
        "pa_pool_incr_ref": ([P, I32], I),
        "pa_pool_ref": ([P, I32], I),
        "pa_pool_seq_new": ([P, ctypes.POINTER(I64)], I),
        "pa_pool_seq_fork": ([P, I64, ctypes.POINTER(I64)], I),
        "pa_pool_seq_share_prefix": ([P, I64, P, I, I64], I),
        "pa_pool_seq_append": ([P, I64, ctypes.POINTER(I64), ctypes.POINTER(I32),
                                ctypes.POINTER(I32)], I),
        "pa_pool_seq_free": ([P, I64], I),
        "pa_pool_seq_append_batch": ([P, P, I, P, P, ctypes.POINTER(I)], I),
        "pa_pool_seq_len": ([P, I64], I64),
        "pa_pool_build_block_tables": ([P, P, I, I, P, P], I),
        "pa_pool_stats": ([P, ctypes.POINTER(_Stats)], I),
        "pa_pool_seq_blocks": ([P, I64, P, I, ctypes.POINTER(I)], I),
        "pa_pool_step": ([P, P, I, I, P, P, ctypes.POINTER(I), P, P], I),
        "pa_pool_cache_block": ([P, I32, ctypes.c_uint64, ctypes.POINTER(I)], I),
        "pa_pool_cache_lookup": ([P, ctypes.c_uint64, ctypes.POINTER(I32)], I),
        "pa_pool_seq_match_prefix": ([P, I64, P, I, ctypes.POINTER(I)], I),
        "pa_plan_shards": ([P, I, I, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def pa_last_error() -> str:
    return lib().pa_last_error().decode()


def _check(st: int) -> None:
    if st != 0:
        raise PaError(st, pa_last_error())


def pa_version() -> int:
    return lib().pa_version()


def pa_launch_count() -> int:
    """Kernels the library has enqueued in this process (all devices, streams)."""
    return int(lib().pa_launch_count())


_CUDA_AVAILABLE = None


def _stream(stream) -> ctypes.c_void_p:
    global _CUDA_AVAILABLE
    if stream is None:
        if _CUDA_AVAILABLE is None:
            _CUDA_AVAILABLE = torch.cuda.is_available()
        if not _CUDA_AVAILABLE:                 # host-only calls (argument checks)
            return ctypes.c_void_p(0)
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _dt(t: torch.Tensor) -> int:
    try:
        return _TORCH_DT[t.dtype]
    except KeyError:
        raise PaError(1, f"unsupported dtype {t.dtype}") from None


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise PaError(1, "tensors must be contiguous")
    return t.data_ptr()


def pa_device_status(clear: bool = True, stream=None) -> int:
    """Sticky device error bits (PA_DEV_*); synchronises the stream."""
    bits = ctypes.c_uint(0)
    _check(lib().pa_device_status(ctypes.byref(bits), int(clear), _stream(stream)))
    return bits.value


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                         k_scale: float = 1.0, v_scale: float = 1.0, stream=None) -> None:
    """key/value [T, Hkv, D]; caches [NB, bs, Hkv, D]; slot_mapping [T] int64."""
    T, Hkv, D = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[1]
    if slot_mapping.dtype != torch.int64:
        raise PaError(1, "slot_mapping must be int64")
    _check(lib().pa_reshape_and_cache(_ptr(key), _ptr(value), _dt(key), _ptr(key_cache),
                                      _ptr(value_cache), _dt(key_cache), _ptr(slot_mapping),
                                      T, Hkv, D, bs, NB, float(k_scale), float(v_scale),
                                      _stream(stream)))


def pa_copy_blocks(key_cache: torch.Tensor, value_cache: torch.Tensor, pairs,
                   stream=None) -> None:
    """pairs: host [n, 2] int32 (src, dst) -- a CPU tensor, array or list of pairs."""
    pr = torch.as_tensor(pairs, dtype=torch.int32).reshape(-1, 2).contiguous()
    if pr.device.type != "cpu":
        raise PaError(1, "pairs live in host memory")
    NB = key_cache.shape[0]
    block_bytes = key_cache[0].numel() * key_cache.element_size() if NB else 0
    _check(lib().pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), block_bytes, NB,
                                pr.data_ptr() if pr.numel() else None, pr.shape[0],
                                _stream(stream)))


def pa_decode_workspace_size(S: int, Hq: int, D: int, max_ctx: int, partition: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().pa_decode_workspace_size(S, Hq, D, max_ctx, partition, ctypes.byref(n)))
    return n.value


def pa_decode_suggest_partition(Hkv: int, block_size: int, context_lens_host) -> int:
    cl = torch.as_tensor(context_lens_host, dtype=torch.int32).contiguous()
    out = ctypes.c_int(0)
    _check(lib().pa_decode_suggest_partition(cl.numel(), Hkv, block_size,
                                             cl.data_ptr() if cl.numel() else None,
                                             ctypes.byref(out)))
    return out.value


def pa_decode_partition_group(S: int, Hq: int, Hkv: int, D: int, block_size: int, q_dtype,
                              cache_dtype, max_ctx: int, partition: int, num_sms: int = 0) -> int:
    """Consecutive split-K partitions one pa_decode CTA streams for this shape
    (planned; each partition keeps its own record)."""
    def code(t):
        return _TORCH_DT[t] if isinstance(t, torch.dtype) else int(t)
    out = ctypes.c_int(0)
    _check(lib().pa_decode_partition_group(S, Hq, Hkv, D, block_size, code(q_dtype),
                                           code(cache_dtype), max_ctx, partition, num_sms,
                                           ctypes.byref(out)))
    return out.value


DECODE_SIMT_ONLY, DECODE_EVICT_FIRST, DECODE_PARTITION_MAJOR = 1, 2, 4
DECODE_GROUP_PARTITIONS = 8
DECODE_SUFFIX_PERSISTENT = 16
DECODE_ONE_HEAD_PER_CTA = 32
PREFILL_CTA_PAIRS = 64
DECODE_DEFAULT = DECODE_PARTITION_MAJOR
PA_PARTITION_BALANCED = -1                        # include/pa.h: the persistent balanced grid
PA_DECODE_NOALLOC_SCRATCH_BYTES = 32 << 20        # include/pa.h: pa_decode_noalloc's array


def pa_decode_select(mode: int) -> None:
    """Bit mask: 1 CUDA-core consumer everywhere, 2 L2 evict-first K/V loads,
    4 partition-major grid, 8 split-K partitions grouped three to a CTA whenever
    there are several, 16 shared-prefix decode with the persistent whole-item
    grid for the suffixes instead of one CTA per (sequence, kv head) suffix,
    32 one kv head per CTA everywhere instead of groups of four (default 4)."""
    _check(lib().pa_decode_select(int(mode)))


def pa_decode(out: torch.Tensor, q: torch.Tensor, key_cache: torch.Tensor,
              value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
              max_ctx: int, scale: float, k_scale: float = 1.0, v_scale: float = 1.0,
              partition: int = 0, workspace: Optional[torch.Tensor] = None,
              stream=None) -> None:
    """out/q [S, Hq, D]; caches [NB, bs, Hkv, D]; block_tables [S, MB] int32;
    context_lens [S] int32; workspace: device bytes >= pa_decode_workspace_size()."""
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PaError(1, "block_tables and context_lens must be int32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode(_ptr(out), _ptr(q), _dt(q), _ptr(key_cache), _ptr(value_cache),
                           _dt(key_cache), _ptr(block_tables), MB, _ptr(context_lens), S, Hq,
                           Hkv, D, bs, NB, int(max_ctx), float(scale), float(k_scale),
                           float(v_scale), int(partition), _ptr(workspace), ws_bytes,
                           _stream(stream)))


def pa_decode_noalloc(out: torch.Tensor, q: torch.Tensor, key_cache: torch.Tensor,
                      value_cache: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, max_ctx: int, scale: float,
                      k_scale: float = 1.0, v_scale: float = 1.0, partition: int = 0,
                      stream=None) -> None:
    """pa_decode for callers that cannot allocate device memory: the split-K
    partials go to the library's built-in scratch array (see include/pa.h for
    its size and for the rule that calls overlapping on the GPU race on it)."""
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PaError(1, "block_tables and context_lens must be int32")
    _check(lib().pa_decode_noalloc(_ptr(out), _ptr(q), _dt(q), _ptr(key_cache),
                                   _ptr(value_cache), _dt(key_cache), _ptr(block_tables), MB,
                                   _ptr(context_lens), S, Hq, Hkv, D, bs, NB, int(max_ctx),
                                   float(scale), float(k_scale), float(v_scale), int(partition),
                                   _stream(stream)))


def pa_decode_shared_prefix_workspace_size(S: int, Hq: int, Hkv: int, D: int, bs: int,
                                           max_ctx: int, prefix_tokens: int, cache_dtype) -> int:
    n = ctypes.c_size_t()
    dt = _TORCH_DT[cache_dtype] if isinstance(cache_dtype, torch.dtype) else int(cache_dtype)
    _check(lib().pa_decode_shared_prefix_workspace_size(S, Hq, Hkv, D, bs, int(max_ctx),
                                                         int(prefix_tokens), dt, ctypes.byref(n)))
    return n.value


def pa_decode_shared_prefix(out: torch.Tensor, q: torch.Tensor, key_cache: torch.Tensor,
                            value_cache: torch.Tensor, block_tables: torch.Tensor,
                            context_lens: torch.Tensor, max_ctx: int, scale: float,
                            prefix_tokens: int, workspace: Optional[torch.Tensor],
                            k_scale: float = 1.0, v_scale: float = 1.0, stream=None) -> None:
    """pa_decode for a batch whose tables start with the same prefix blocks (row
    0's first prefix_tokens / bs): the prefix is attended once for all queries."""
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise PaError(1, "block_tables and context_lens must be int32")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_shared_prefix(_ptr(out), _ptr(q), _dt(q), _ptr(key_cache),
                                         _ptr(value_cache), _dt(key_cache), _ptr(block_tables),
                                         MB, _ptr(context_lens), S, Hq, Hkv, D, bs, NB,
                                         int(max_ctx), float(scale), float(k_scale),
                                         float(v_scale), int(prefix_tokens), _ptr(workspace),
                                         ws_bytes, _stream(stream)))


def pa_prefill(out: torch.Tensor, q: torch.Tensor, key_cache: torch.Tensor,
               value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
               query_start: torch.Tensor, max_query_len: int, scale: float,
               stream=None) -> None:
    """Causal attention of a batch of new-token chunks over the paged cache.
    out/q [T, Hq, D]; caches [NB, bs, Hkv, D] (same dtype as q); block_tables
    [S, MB] int32; context_lens [S] int32 (cached + new tokens); query_start
    [S + 1] int32 (row offsets of each sequence's new tokens in q)."""
    T, Hq, D = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    S = context_lens.numel()
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    for t in (block_tables, context_lens, query_start):
        if t.dtype != torch.int32:
            raise PaError(1, "block_tables, context_lens and query_start must be int32")
    if query_start.numel() != S + 1:
        raise PaError(1, "query_start must hold S + 1 offsets")
    _check(lib().pa_prefill(_ptr(out), _ptr(q), _dt(q), _ptr(key_cache), _ptr(value_cache),
                            _dt(key_cache), _ptr(block_tables), MB, _ptr(context_lens),
                            _ptr(query_start), S, T, Hq, Hkv, D, bs, NB, int(max_query_len),
                            float(scale), _stream(stream)))


def pa_plan_shards(context_lens, ndev: int):
    """Split a batch over ndev GPUs by sequence (host): -> (device of each
    sequence int32 [S], tokens per device int64 [ndev]).  Longest first, each to
    the device with the fewest tokens so far."""
    lens = torch.as_tensor(context_lens, dtype=torch.int32).cpu().contiguous()
    S = lens.numel()
    dev = torch.empty(S, dtype=torch.int32)
    tok = torch.empty(max(int(ndev), 1), dtype=torch.int64)
    _check(lib().pa_plan_shards(lens.data_ptr() if S else None, S, int(ndev),
                                dev.data_ptr() if S else None, tok.data_ptr()))
    return dev, tok


class BlockPool:
    """Host refcounted block pool (pa_pool_*): FIFO free queue, per-sequence
    block tables, sharing and copy-on-write decisions.  Not thread-safe."""

    def __init__(self, num_blocks: int, block_size: int):
        self._p = ctypes.c_void_p()
        _check(lib().pa_pool_create(num_blocks, block_size, ctypes.byref(self._p)))
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._p:
            lib().pa_pool_destroy(self._p)
            self._p = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown
            pass

    def alloc(self) -> int:
        b = ctypes.c_int32()
        _check(lib().pa_pool_alloc(self._p, ctypes.byref(b)))
        return b.value

    def free(self, block: int) -> None:
        _check(lib().pa_pool_free(self._p, block))

    def incr_ref(self, block: int) -> None:
        _check(lib().pa_pool_incr_ref(self._p, block))

    def ref(self, block: int) -> int:
        return lib().pa_pool_ref(self._p, block)

    def seq_new(self) -> int:
        s = ctypes.c_int64()
        _check(lib().pa_pool_seq_new(self._p, ctypes.byref(s)))
        return s.value

    def seq_fork(self, parent: int) -> int:
        s = ctypes.c_int64()
        _check(lib().pa_pool_seq_fork(self._p, parent, ctypes.byref(s)))
        return s.value

    def seq_share_prefix(self, seq: int, blocks: Sequence[int], num_tokens: int) -> None:
        arr = (ctypes.c_int32 * len(blocks))(*blocks)
        _check(lib().pa_pool_seq_share_prefix(self._p, seq, arr, len(blocks), num_tokens))

    def seq_append(self, seq: int):
        """-> (slot, cow_src, cow_dst); cow_* are -1 when no copy is needed."""
        slot, src, dst = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_pool_seq_append(self._p, seq, ctypes.byref(slot), ctypes.byref(src),
                                        ctypes.byref(dst)))
        return slot.value, src.value, dst.value

    def seq_append_batch(self, seqs, slots_out: Optional[torch.Tensor] = None,
                         cow_out: Optional[torch.Tensor] = None):
        """Append one token to each sequence: -> (slots int64 [n], cow pairs int32 [k, 2]).
        seqs: host int64 tensor or sequence; outputs may be preallocated host tensors."""
        ids = torch.as_tensor(seqs, dtype=torch.int64).contiguous()
        n = ids.numel()
        if slots_out is None:
            slots_out = torch.empty(n, dtype=torch.int64)
        if cow_out is None:
            cow_out = torch.empty((max(n, 1), 2), dtype=torch.int32)
        nc = ctypes.c_int(0)
        _check(lib().pa_pool_seq_append_batch(self._p, ids.data_ptr() if n else None, n,
                                              slots_out.data_ptr() if n else None,
                                              cow_out.data_ptr(), ctypes.byref(nc)))
        return slots_out, cow_out[:nc.value]

    def seq_free(self, seq: int) -> None:
        _check(lib().pa_pool_seq_free(self._p, seq))

    def seq_len(self, seq: int) -> int:
        return lib().pa_pool_seq_len(self._p, seq)

    def build_block_tables(self, seqs: Sequence[int], max_blocks: int,
                           tables_out: Optional[torch.Tensor] = None,
                           lens_out: Optional[torch.Tensor] = None):
        """Pack the tables into host int32 [S, max_blocks] (-1 padded) + lens [S]."""
        if isinstance(seqs, torch.Tensor):
            assert seqs.dtype == torch.int64 and seqs.device.type == "cpu" and seqs.is_contiguous()
            S = seqs.numel()
            ids = ctypes.c_void_p(seqs.data_ptr()) if S else None
        else:
            S = len(seqs)
            ids = (ctypes.c_int64 * S)(*seqs)
        if tables_out is None:
            tables_out = torch.empty((S, max_blocks), dtype=torch.int32)
        if lens_out is None:
            lens_out = torch.empty((S,), dtype=torch.int32)
        assert tables_out.device.type == "cpu" and lens_out.device.type == "cpu"
        _check(lib().pa_pool_build_block_tables(self._p, ids, S, max_blocks,
                                                 tables_out.data_ptr() if tables_out.numel() else None,
                                                 lens_out.data_ptr() if S else None))
        return tables_out, lens_out

    def stats(self) -> dict:
        st = _Stats()
        _check(lib().pa_pool_stats(self._p, ctypes.byref(st)))
        return {n: getattr(st, n) for n, _ in _Stats._fields_}

    def step(self, seqs: torch.Tensor, max_blocks: int, slots_out: torch.Tensor,
             cow_out: torch.Tensor, tables_out: torch.Tensor, lens_out: torch.Tensor):
        """One decode step's host work: append a token to every sequence of the
        contiguous host int64 tensor `seqs` and pack their tables and lengths
        into the given host tensors.  -> copy-on-write pairs int32 [k, 2]."""
        n = seqs.numel()
        nc = ctypes.c_int(0)
        _check(lib().pa_pool_step(self._p, seqs.data_ptr() if n else None, n, max_blocks,
                                  slots_out.data_ptr() if n else None, cow_out.data_ptr(),
                                  ctypes.byref(nc),
                                  tables_out.data_ptr() if tables_out.numel() else None,
                                  lens_out.data_ptr() if n else None))
        return cow_out[:nc.value]

    def seq_blocks(self, seq: int) -> list:
        n = ctypes.c_int(0)
        lib().pa_pool_seq_blocks(self._p, seq, None, 0, ctypes.byref(n))   # size query
        arr = (ctypes.c_int32 * max(n.value, 1))()
        _check(lib().pa_pool_seq_blocks(self._p, seq, arr, n.value, ctypes.byref(n)))
        return list(arr[:n.value])

    # -- prefix cache (content hashes of full blocks) ---------------------------
    def cache_block(self, block: int, content_hash: int) -> bool:
        """Register a full, in-use block as holding ``content_hash`` (uint64).
        True if it is now the block for that hash, False if another block is."""
        c = ctypes.c_int(0)
        _check(lib().pa_pool_cache_block(self._p, block, content_hash & 0xFFFFFFFFFFFFFFFF,
                                         ctypes.byref(c)))
        return bool(c.value)

    def cache_lookup(self, content_hash: int) -> int:
        """The cached block for the hash with one more reference taken, or -1."""
        b = ctypes.c_int32()
        _check(lib().pa_pool_cache_lookup(self._p, content_hash & 0xFFFFFFFFFFFFFFFF,
                                          ctypes.byref(b)))
        return b.value

    def seq_match_prefix(self, seq: int, hashes: Sequence[int]) -> int:
        """An empty sequence takes the cached blocks of the leading hashes that
        hit; returns how many matched (it then holds that many full blocks)."""
        arr = (ctypes.c_uint64 * max(len(hashes), 1))(*[h & 0xFFFFFFFFFFFFFFFF for h in hashes])
        m = ctypes.c_int(0)
        _check(lib().pa_pool_seq_match_prefix(self._p, seq, arr, len(hashes), ctypes.byref(m)))
        return m.value
