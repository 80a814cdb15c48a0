"""pa_decode_noalloc against pa_decode (GPU).

pa_decode_noalloc serves callers that cannot allocate device memory (a runtime
that owns all of it, a plugin without an allocation hook, a step loop that may
not call cudaMalloc/cudaFree): its split-K partials live in the library's
built-in scratch array instead of a caller workspace.  This file is collected
last on purpose, so that a run stopping at its first failure has run every
other test first.  It is self-contained: it passes alone in a fresh process
and after the rest of the suite.
"""
import pytest
import torch

import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-2   # bf16 cache, the same bar as the oracle parity tests


def _inputs(seed):
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 8, 200, 1500)
    inp = wl.make_decode_inputs(cfg, seed=seed)
    d = {k: getattr(inp, k).cuda() for k in
         ("q", "key_cache", "value_cache", "key_new", "value_new", "slot_mapping",
          "block_tables", "context_lens")}
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], d["key_cache"], d["value_cache"],
                            d["slot_mapping"])
    return inp, d


def test_noalloc_matches_decode_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    part = 128                                   # several partitions per sequence: scratch in use
    for seed in (31, 32):                        # two calls in a row, different data
        inp, d = _inputs(seed)
        S, Hq, D = d["q"].shape
        need = pa.pa_decode_workspace_size(S, Hq, D, inp.max_ctx, part)
        assert 0 < need <= (32 << 20)
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(d["q"])
        pa.pa_decode(ref, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                     d["context_lens"], inp.max_ctx, inp.scale, partition=part, workspace=ws)
        got = torch.full_like(d["q"], float("nan"))
        pa.pa_decode_noalloc(got, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                             d["context_lens"], inp.max_ctx, inp.scale, partition=part)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        err = (got.float() - ref.float()).abs().max().item()
        assert err <= TOL, err
    assert pa.pa_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    inp, d = _inputs(33)
    S, Hq, D = d["q"].shape
    huge_ctx = 4_000_000            # 8 seqs x 32 heads x 250k partitions of 16: far past 32 MiB
    assert pa.pa_decode_workspace_size(S, Hq, D, huge_ctx, 16) > (32 << 20)
    out = torch.empty_like(d["q"])
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(out, d["q"], d["key_cache"], d["value_cache"], d["block_tables"],
                             d["context_lens"], huge_ctx, inp.scale, partition=16)
    assert e.value.status == "PA_ERR_INVALID_ARG" and "scratch" in str(e.value)
