"""The oracle -- TEST INFRASTRUCTURE ONLY.

Plain fp64 CPU statements of what the paged-decode path computes (``pa_oracle.c``)
and of how the refcounted block pool behaves (``pool_model.py``).  Only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package.  It shares no code with the CUDA library and never imports it.

Every function takes host arrays (numpy, or CPU torch tensors, which are viewed
as their raw bytes) and dtype names "f32", "f16", "bf16", "fp8_e4m3".

Parity status of each part (what pins it, see tests/test_oracle_*.py):
  prefill attention  -- pinned: torch SDPA in float64 with an explicit causal
                        mask on the unpaged gather, L=1 rows = decode rows,
                        chunk invariance (one chunk = two chunks), causality
                        (keys past a row's position do not change it), the
                        first token of a prefill returns v_0.
  decode attention   -- pinned: torch SDPA in float64 on the unpaged gather,
                        brute force on tiny cases, invariants (block-id
                        permutation, shared prefix, weights sum to 1) and the
                        closed-form special cases (n=1, q=0, a dominant logit,
                        GQA = replicated MHA).
  storage decoders   -- pinned: numpy float16 / torch bfloat16 / torch float8
                        conversions and the OCP E4M3 value table's closed forms.
  E4M3 encoder       -- pinned: torch float8_e4m3fn conversion inside the range,
                        every midpoint (ties to even), saturation.
  cache append, copy -- pinned: byte placement checked against slot arithmetic
                        done by hand in the tests; copy against numpy indexing.
  pool model         -- pinned: the block-table and refcount examples printed on
                        "01. PagedAttention 详解" §3 and §6 (tests/golden/).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libpa_oracle.so")

DT = {"f32": 0, "f16": 1, "bf16": 2, "fp8_e4m3": 3}
_ESIZE = {"f32": 4, "f16": 2, "bf16": 2, "fp8_e4m3": 1}
_RAWNP = {4: np.uint32, 2: np.uint16, 1: np.uint8}
ERRORS = {-1: "invalid argument", -2: "index out of range", -3: "out of memory"}


def build(force: bool = False) -> str:
    """Compile pa_oracle.c with gcc (no fast-math: IEEE binary64 arithmetic)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        P, I, I64, D, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
        L.orc_f32_value.restype = D
        L.orc_f32_value.argtypes = [ctypes.c_uint32]
        L.orc_f16_value.restype = D
        L.orc_f16_value.argtypes = [ctypes.c_uint16]
        L.orc_bf16_value.restype = D
        L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_value.restype = D
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_values.argtypes = [P, P, I, SZ]
        L.orc_values.restype = None
        L.orc_e4m3_encode_array.argtypes = [P, P, SZ]
        L.orc_e4m3_encode_array.restype = None
        L.orc_reshape_and_cache.argtypes = [P, P, I, P, P, I, P, I, I, I, I, I64,
                                            ctypes.c_float, ctypes.c_float]
        L.orc_reshape_and_cache.restype = I
        L.orc_copy_blocks.argtypes = [P, P, SZ, I64, P, I]
        L.orc_copy_blocks.restype = I
        L.orc_paged_decode.argtypes = [P, P, I, P, P, I, P, I, P, I, I, I, I, I, I64,
                                       D, D, D, P, I, I]
        L.orc_paged_decode.restype = I
        L.orc_decode_weights.argtypes = [P, P, I, P, I, P, I, P, I, I, I, I, I64, D, D, I, I]
        L.orc_decode_weights.restype = I
        L.orc_paged_prefill.argtypes = [P, P, I, P, P, I, P, I, P, P, I, I, I, I, I, I, I64,
                                        D, D, D, P, I, I]
        L.orc_paged_prefill.restype = I
    return _lib


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: {ERRORS.get(rc, rc)}")


def raw(x, dtype: str | None = None) -> np.ndarray:
    """Contiguous numpy view of the raw storage of a CPU tensor or ndarray."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            assert x.device.type == "cpu", "the oracle takes host tensors"
            x = x.contiguous()
            if x.dtype in (torch.bfloat16, torch.float16, torch.float32, torch.float8_e4m3fn):
                x = x.view({4: torch.int32, 2: torch.int16, 1: torch.uint8}[x.element_size()])
            return np.ascontiguousarray(x.numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def values(x, dtype: str) -> np.ndarray:
    """Decode stored values of ``dtype`` to float64 (same shape)."""
    a = raw(x)
    out = np.empty(a.shape, dtype=np.float64)
    lib().orc_values(_ptr(out), _ptr(a), DT[dtype], a.size)
    return out


def e4m3_encode(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_ptr(out), _ptr(a), a.size)
    return out


def reshape_and_cache(key, value, in_dtype, key_cache, value_cache, cache_dtype,
                      slot_mapping, block_size, k_scale=1.0, v_scale=1.0):
    """Return (key_cache', value_cache') as raw numpy arrays after the append."""
    k, v = raw(key), raw(value)
    kc, vc = raw(key_cache).copy(), raw(value_cache).copy()
    sm = np.ascontiguousarray(np.asarray(raw(slot_mapping), dtype=np.int64))
    T, Hkv, D = k.shape
    NB = kc.shape[0]
    rc = lib().orc_reshape_and_cache(_ptr(k), _ptr(v), DT[in_dtype], _ptr(kc), _ptr(vc),
                                     DT[cache_dtype], _ptr(sm), T, Hkv, D, block_size, NB,
                                     float(k_scale), float(v_scale))
    _check(rc, "reshape_and_cache")
    return kc, vc


def copy_blocks(key_cache, value_cache, pairs):
    """Return (key_cache', value_cache') with whole blocks copied src -> dst."""
    kc, vc = raw(key_cache).copy(), raw(value_cache).copy()
    pr = np.ascontiguousarray(np.asarray(raw(pairs), dtype=np.int32).reshape(-1, 2))
    NB = kc.shape[0]
    block_bytes = kc[0].nbytes
    rc = lib().orc_copy_blocks(_ptr(kc), _ptr(vc), block_bytes, NB, _ptr(pr), pr.shape[0])
    _check(rc, "copy_blocks")
    return kc, vc


def paged_decode(q, q_dtype, key_cache, value_cache, kv_dtype, block_tables, context_lens,
                 scale, k_scale=1.0, v_scale=1.0, seqs=None, nthreads=0) -> np.ndarray:
    """fp64 attention output [len(seqs) or S, Hq, D]."""
    qa = raw(q)
    kc, vc = raw(key_cache), raw(value_cache)
    bt = np.ascontiguousarray(np.asarray(raw(block_tables), dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(raw(context_lens), dtype=np.int32))
    S, Hq, D = qa.shape
    NB, bs, Hkv, D2 = kc.shape
    assert D2 == D
    MB = bt.shape[1] if bt.ndim == 2 else 0
    sel = None if seqs is None else np.ascontiguousarray(np.asarray(seqs, dtype=np.int32))
    nsel = S if sel is None else sel.size
    out = np.zeros((nsel, Hq, D), dtype=np.float64)
    rc = lib().orc_paged_decode(_ptr(out), _ptr(qa), DT[q_dtype], _ptr(kc), _ptr(vc),
                                DT[kv_dtype], _ptr(bt), MB, _ptr(cl), S, Hq, Hkv, D, bs, NB,
                                float(scale), float(k_scale), float(v_scale),
                                None if sel is None else _ptr(sel), nsel, int(nthreads))
    _check(rc, "paged_decode")
    return out


def decode_weights(q, q_dtype, key_cache, kv_dtype, block_tables, context_lens, scale,
                   s, h, k_scale=1.0) -> np.ndarray:
    """Normalised softmax weights w[0..n_s) of sequence s, query head h."""
    qa, kc = raw(q), raw(key_cache)
    bt = np.ascontiguousarray(np.asarray(raw(block_tables), dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(raw(context_lens), dtype=np.int32))
    S, Hq, D = qa.shape
    NB, bs, Hkv, _ = kc.shape
    w = np.zeros(max(int(cl[s]), 1), dtype=np.float64)
    rc = lib().orc_decode_weights(_ptr(w), _ptr(qa), DT[q_dtype], _ptr(kc), DT[kv_dtype],
                                  _ptr(bt), bt.shape[1], _ptr(cl), Hq, Hkv, D, bs, NB,
                                  float(scale), float(k_scale), int(s), int(h))
    _check(rc, "decode_weights")
    return w[:int(cl[s])]


def paged_prefill(q, q_dtype, key_cache, value_cache, kv_dtype, block_tables, context_lens,
                  query_start, scale, k_scale=1.0, v_scale=1.0, rows=None,
                  nthreads=0) -> np.ndarray:
    """fp64 causal attention of the new tokens [len(rows) or T, Hq, D]."""
    qa = raw(q)
    kc, vc = raw(key_cache), raw(value_cache)
    bt = np.ascontiguousarray(np.asarray(raw(block_tables), dtype=np.int32))
    cl = np.ascontiguousarray(np.asarray(raw(context_lens), dtype=np.int32))
    qs = np.ascontiguousarray(np.asarray(raw(query_start), dtype=np.int32))
    T, Hq, D = qa.shape
    NB, bs, Hkv, D2 = kc.shape
    assert D2 == D
    S = cl.size
    MB = bt.shape[1] if bt.ndim == 2 else 0
    sel = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    nrow = T if sel is None else sel.size
    out = np.zeros((nrow, Hq, D), dtype=np.float64)
    rc = lib().orc_paged_prefill(_ptr(out), _ptr(qa), DT[q_dtype], _ptr(kc), _ptr(vc),
                                 DT[kv_dtype], _ptr(bt), MB, _ptr(cl), _ptr(qs), S, T, Hq, Hkv,
                                 D, bs, NB, float(scale), float(k_scale), float(v_scale),
                                 None if sel is None else _ptr(sel), nrow, int(nthreads))
    _check(rc, "paged_prefill")
    return out
