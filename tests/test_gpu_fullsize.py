"""GPU parity of the decode step at the benchmark workloads' full sizes, in the
launch configuration bench.py times, on sequences the oracle computes one by
one.

Each case builds the workload exactly as the bench does (seed 2, every
sequence, the whole cache), runs the step on the GPU through the C ABI --
copy-on-write copies, the append, then pa_decode with the partition bench.py
uses (the workload's stated split, else pa_decode_suggest_partition), or
pa_decode_shared_prefix for the shared-prefix workload -- and compares sampled
sequences (the first, the last, the longest and two drawn at random) with the
fp64 oracle's own copy, append and attention.  Bars as in test_gpu_parity.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2}
FULL = [("llama2_7b_mha_fp16_b64", 0), ("llama3_8b_gqa_bf16_b128", 0),
        ("long_context_splitk_bf16_4x100k", 0), ("prefix_shared_fp8_b256", 0),
        # the Llama-3-8B shape at the other block sizes (bench.py --block-size)
        ("llama3_8b_gqa_bf16_b128", 8), ("llama3_8b_gqa_bf16_b128", 32)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    pa.pa_decode_select(pa.DECODE_DEFAULT)
    yield


def _oracle(inp: wl.DecodeInputs, seqs):
    cfg = inp.cfg
    kc, vc = inp.key_cache, inp.value_cache
    if inp.copy_pairs.numel():
        k2, v2 = oracle.copy_blocks(kc, vc, inp.copy_pairs)
        kc = torch.from_numpy(k2).view(kc.dtype).reshape(kc.shape)
        vc = torch.from_numpy(v2).view(vc.dtype).reshape(vc.shape)
    k3, v3 = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.q_dtype, kc, vc,
                                      cfg.kv_dtype, inp.slot_mapping, cfg.block_size,
                                      inp.k_scale, inp.v_scale)
    kc = torch.from_numpy(k3).view(kc.dtype).reshape(kc.shape)
    vc = torch.from_numpy(v3).view(vc.dtype).reshape(vc.shape)
    return oracle.paged_decode(inp.q, cfg.q_dtype, kc, vc, cfg.kv_dtype, inp.block_tables,
                               inp.context_lens, inp.scale, inp.k_scale, inp.v_scale, seqs=seqs)


@pytest.mark.parametrize("name,bs", FULL, ids=[f"{n}_bs{b}" if b else n for n, b in FULL])
def test_full_size_sampled(name, bs):
    cfg = wl.DECODE_WORKLOADS[name]
    if bs:
        cfg = dataclasses.replace(cfg, block_size=bs, name=f"{name}_bs{bs}")
    inp = wl.make_decode_inputs(cfg, seed=2)
    S, Hq, D = inp.q.shape
    lens = inp.context_lens
    d = {k: getattr(inp, k).cuda() for k in ("q", "key_cache", "value_cache", "key_new",
                                              "value_new", "slot_mapping", "block_tables",
                                              "context_lens")}
    kc, vc = d["key_cache"], d["value_cache"]
    if inp.copy_pairs.numel():
        pa.pa_copy_blocks(kc, vc, inp.copy_pairs)
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], kc, vc, d["slot_mapping"],
                            inp.k_scale, inp.v_scale)
    out = torch.full_like(d["q"], float("nan"))
    pa.pa_device_status(clear=True)
    if cfg.prefix_tokens:
        nb = pa.pa_decode_shared_prefix_workspace_size(S, Hq, cfg.num_kv_heads, D, cfg.block_size,
                                                       inp.max_ctx, cfg.prefix_tokens, kc.dtype)
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
        pa.pa_decode_shared_prefix(out, d["q"], kc, vc, d["block_tables"], d["context_lens"],
                                   inp.max_ctx, inp.scale, cfg.prefix_tokens, ws if nb else None,
                                   inp.k_scale, inp.v_scale)
    else:
        part = cfg.partition or pa.pa_decode_suggest_partition(cfg.num_kv_heads,
                                                               cfg.block_size, lens)
        nb = pa.pa_decode_workspace_size(S, Hq, D, inp.max_ctx, part)
        ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
        pa.pa_decode(out, d["q"], kc, vc, d["block_tables"], d["context_lens"], inp.max_ctx,
                     inp.scale, inp.k_scale, inp.v_scale, part, ws if nb else None)
    torch.cuda.synchronize()
    assert pa.pa_device_status() == 0
    g = torch.Generator().manual_seed(len(name))
    seqs = sorted({0, S - 1, int(lens.argmax())} |
                  set(torch.randint(0, S, (2,), generator=g).tolist()))
    want = _oracle(inp, seqs)
    got = out[seqs].cpu().to(torch.float64).numpy()
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - want).max()
    assert err <= TOL[cfg.kv_dtype], f"{name}: max abs error {err:.3g} on sequences {seqs}"
