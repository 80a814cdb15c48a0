"""pa_decode_noalloc against pa_decode and the oracle (GPU).

pa_decode_noalloc serves callers that cannot allocate device memory (a runtime
that owns all of it, a plugin without an allocation hook, a step loop that may
not call cudaMalloc/cudaFree): its split-K partials live in the library's
built-in scratch array instead of a caller workspace.  It runs the same
kernels with the same plan as pa_decode, so the two outputs must be
bit-identical; both are also held to the oracle's bf16 bar.  The scratch
array keeps the previous call's contents, so the persistent balanced grid
(whose merge reads per-item CTA records from it) is run right after a call
with another batch size, over scratch full of stale records.

This file is collected last on purpose, so that a run stopping at its first
failure has run every other test first.  It is self-contained: it passes alone
in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-2   # bf16 cache: the decode bar of the oracle parity tests


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


def _inputs(seed, nseq=8):
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], nseq, 200, 1500)
    inp = wl.make_decode_inputs(cfg, seed=seed)
    d = {k: getattr(inp, k).cuda() for k in
         ("q", "key_cache", "value_cache", "key_new", "value_new", "slot_mapping",
          "block_tables", "context_lens")}
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], d["key_cache"], d["value_cache"],
                            d["slot_mapping"])
    return inp, d


def _reference(inp, d, part):
    """pa_decode with a workspace of its own, filled with garbage first."""
    S, Hq, D = d["q"].shape
    need = pa.pa_decode_workspace_size(S, Hq, D, inp.max_ctx, part)
    assert 0 < need <= pa.PA_DECODE_NOALLOC_SCRATCH_BYTES
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(d["q"])
    pa.pa_decode(ref, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                 d["context_lens"], inp.max_ctx, inp.scale, partition=part, workspace=ws)
    return ref


def _noalloc(inp, d, part):
    got = torch.full_like(d["q"], float("nan"))
    pa.pa_decode_noalloc(got, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                         d["context_lens"], inp.max_ctx, inp.scale, partition=part)
    return got


def _oracle_error(inp, d, got):
    cfg = inp.cfg
    want = oracle.paged_decode(inp.q, cfg.q_dtype, d["key_cache"].cpu(), d["value_cache"].cpu(),
                               cfg.kv_dtype, inp.block_tables, inp.context_lens, inp.scale)
    return np.abs(got.cpu().to(torch.float64).numpy() - want).max()


@pytest.mark.parametrize("part", [128, pa.PA_PARTITION_BALANCED], ids=["split_k", "balanced"])
def test_noalloc_matches_decode_on_two_calls_in_a_row(part):
    # a call with another batch size first: the scratch then holds its records
    inp0, d0 = _inputs(30, nseq=13)
    _noalloc(inp0, d0, 64)
    for seed in (31, 32):                        # two calls in a row, different data
        inp, d = _inputs(seed)
        ref = _reference(inp, d, part)
        got = _noalloc(inp, d, part)
        torch.cuda.synchronize()
        assert pa.pa_device_status() == 0
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref), "pa_decode_noalloc differs from pa_decode"
        err = _oracle_error(inp, d, got)
        assert err <= TOL, f"max abs error {err:.3g} against the oracle"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    inp, d = _inputs(33)
    S, Hq, D = d["q"].shape
    huge_ctx = 4_000_000            # 8 seqs x 32 heads x 250k partitions of 16: far past 32 MiB
    assert pa.pa_decode_workspace_size(S, Hq, D, huge_ctx, 16) > pa.PA_DECODE_NOALLOC_SCRATCH_BYTES
    out = torch.empty_like(d["q"])
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                             d["context_lens"], huge_ctx, inp.scale, partition=16)
    assert e.value.status == "PA_ERR_INVALID_ARG" and "scratch" in str(e.value)
