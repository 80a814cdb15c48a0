"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Bars (stated per dtype of the KV cache, on the attention output, max abs error
against the oracle's double result):  fp32 1e-5, fp16 2e-3, bf16 1e-2,
fp8-e4m3 3e-2.  Cache append and block copy: bit-exact.  Each case runs the
whole decode step -- copy-on-write copies, append, decode (with and without
split-K, with both consumers) -- on seeded inputs from ``workloads`` whose
unused blocks, tail slots and table padding are poisoned (NaN codes / -1).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield
    pa.pa_decode_select(pa.DECODE_DEFAULT)


def _to(inp: wl.DecodeInputs, device):
    f = {}
    for k in ("q", "key_cache", "value_cache", "key_new", "value_new", "slot_mapping",
              "block_tables", "block_tables_pre", "context_lens"):
        f[k] = getattr(inp, k).to(device)
    return f


def gpu_step(inp: wl.DecodeInputs, partition: int, mode: int = pa.DECODE_DEFAULT, max_ctx=None):
    d = _to(inp, "cuda")
    kc, vc = d["key_cache"].clone(), d["value_cache"].clone()
    if inp.copy_pairs.numel():
        pa.pa_copy_blocks(kc, vc, inp.copy_pairs)
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], kc, vc, d["slot_mapping"],
                            inp.k_scale, inp.v_scale)
    out = torch.full_like(d["q"], float("nan"))
    mc = inp.max_ctx if max_ctx is None else max_ctx
    S, Hq, D = d["q"].shape
    ws_bytes = pa.pa_decode_workspace_size(S, Hq, D, mc, partition)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode_select(mode)
    pa.pa_decode(out, d["q"], kc, vc, d["block_tables"], d["context_lens"], mc, inp.scale,
                 inp.k_scale, inp.v_scale, partition, ws if ws_bytes else None)
    torch.cuda.synchronize()
    return out.cpu(), kc.cpu(), vc.cpu()


def oracle_step(inp: wl.DecodeInputs, seqs=None):
    cfg = inp.cfg
    kc, vc = inp.key_cache.cpu(), inp.value_cache.cpu()
    if inp.copy_pairs.numel():
        k2, v2 = oracle.copy_blocks(kc, vc, inp.copy_pairs)
        kc = torch.from_numpy(k2).view(kc.dtype).reshape(kc.shape)
        vc = torch.from_numpy(v2).view(vc.dtype).reshape(vc.shape)
    k3, v3 = oracle.reshape_and_cache(inp.key_new.cpu(), inp.value_new.cpu(), cfg.q_dtype, kc, vc,
                                      cfg.kv_dtype, inp.slot_mapping.cpu(), cfg.block_size,
                                      inp.k_scale, inp.v_scale)
    kc = torch.from_numpy(k3).view(kc.dtype).reshape(kc.shape)
    vc = torch.from_numpy(v3).view(vc.dtype).reshape(vc.shape)
    out = oracle.paged_decode(inp.q.cpu(), cfg.q_dtype, kc, vc, cfg.kv_dtype,
                              inp.block_tables.cpu(), inp.context_lens.cpu(), inp.scale,
                              inp.k_scale, inp.v_scale, seqs=seqs)
    return out, kc, vc


def _bits_equal(a: torch.Tensor, b: torch.Tensor, dt: str) -> bool:
    return torch.equal(wl.raw_view(a.contiguous(), dt), wl.raw_view(b.contiguous(), dt))


def _check_out(got: torch.Tensor, want: np.ndarray, dt: str, what: str):
    g = got.to(torch.float64).numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want).max()
    assert err <= TOL[dt], f"{what}: max abs error {err:.3g} > {TOL[dt]}"
    return err


MODES = [pa.DECODE_DEFAULT, pa.DECODE_DEFAULT | pa.DECODE_SIMT_ONLY,
         pa.DECODE_DEFAULT | pa.DECODE_EVICT_FIRST, 0,
         pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS, pa.DECODE_GROUP_PARTITIONS]
BOTH = [pa.DECODE_DEFAULT, pa.DECODE_DEFAULT | pa.DECODE_SIMT_ONLY]


SMALL = [
    ("tiny_fp32", wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"]),
    ("mha_fp16", wl.small_variant(wl.DECODE_WORKLOADS["llama2_7b_mha_fp16_b64"], 5, 1, 200)),
    ("gqa_bf16", wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 6, 1, 300)),
    ("long_splitk", wl.small_variant(wl.DECODE_WORKLOADS["long_context_splitk_bf16_4x100k"], 2, 1500, 2100)),
    ("prefix_fp8", wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 6, 1, 120, prefix_tokens=64)),
]


@pytest.mark.parametrize("name,cfg", SMALL, ids=[n for n, _ in SMALL])
@pytest.mark.parametrize("partition_blocks", [0, 2, 7, -1], ids=["single", "p2", "p7", "balanced"])
@pytest.mark.parametrize("mode", MODES, ids=["auto", "simt", "evict_first", "head_major",
                                            "grouped", "grouped_head_major"])
def test_step_parity_small(name, cfg, partition_blocks, mode):
    inp = wl.make_decode_inputs(cfg, seed=101)
    want, kc_o, vc_o = oracle_step(inp)
    part = -1 if partition_blocks < 0 else partition_blocks * cfg.block_size
    out, kc, vc = gpu_step(inp, part, mode)
    assert _bits_equal(kc, kc_o, cfg.kv_dtype) and _bits_equal(vc, vc_o, cfg.kv_dtype)
    _check_out(out, want, cfg.kv_dtype, f"{name} P={partition_blocks} mode={mode}")
    assert pa.pa_device_status() == 0


SHAPES = [(bs, G, D, dt) for bs in (8, 16, 32) for G in (1, 2, 4, 8) for D in (64, 128)
          for dt in ("bf16", "f16")] + [(16, 4, 256, "bf16"), (32, 2, 256, "f16"),
                                          (16, 2, 64, "f32"), (8, 4, 128, "fp8_e4m3"),
                                          (32, 8, 256, "fp8_e4m3"), (16, 16, 128, "bf16"),
                                          (8, 16, 64, "f16"), (16, 8, 128, "fp8_e4m3"),
                                          (32, 2, 128, "fp8_e4m3"), (16, 16, 128, "fp8_e4m3"),
                                          (8, 16, 128, "fp8_e4m3")]


@pytest.mark.parametrize("bs,G,D,dt", SHAPES)
def test_decode_shapes(bs, G, D, dt):
    qdt = dt if dt != "fp8_e4m3" else "bf16"
    cfg = wl.DecodeConfig(f"shape_{bs}_{G}_{D}_{dt}", 4, 2 * G, 2, D, bs, dt, qdt, 1,
                          3 * bs + 1, fp8_scaled=dt == "fp8_e4m3")
    inp = wl.make_decode_inputs(cfg, seed=bs * 1000 + G * 10 + D)
    want, _, _ = oracle_step(inp)
    # at block 8, partitions of whole 16-token stages read two blocks a stage
    modes = BOTH + ([pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS] if bs == 8 else [])
    for part in (0, bs, 2 * bs, -1):
        for mode in modes:
            out, _, _ = gpu_step(inp, part, mode)
            _check_out(out, want, dt, f"P={part} mode={mode}")
    assert pa.pa_device_status() == 0


@pytest.mark.parametrize("bs", [16, 8])
@pytest.mark.parametrize("dt", ["bf16", "fp8_e4m3"])
def test_lengths_at_partition_edges(dt, bs):
    P = 64
    lens = (1, P - 1, P, P + 1, 2 * P - 1, 2 * P, 2 * P + 1, 5 * P + 3)
    cfg = wl.DecodeConfig("edges", len(lens), 8, 2, 128, bs, dt, "bf16", 0, 0,
                          fixed_lens=lens, fp8_scaled=dt == "fp8_e4m3")
    inp = wl.make_decode_inputs(cfg, seed=7)
    want, _, _ = oracle_step(inp)
    for mode in BOTH + [pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS]:
        for part in (P, -1):
            out, _, _ = gpu_step(inp, part, mode)
            _check_out(out, want, dt, f"mode={mode} P={part}")


def test_zero_length_sequences_give_zero_rows():
    cfg = wl.DecodeConfig("empty", 3, 8, 2, 128, 16, "bf16", "bf16", 0, 0, fixed_lens=(0, 40, 0))
    inp = wl.make_decode_inputs(cfg, seed=3)
    want, _, _ = oracle_step(inp)
    for part, mode in ((0, pa.DECODE_DEFAULT), (16, pa.DECODE_DEFAULT), (-1, pa.DECODE_DEFAULT),
                       (16, pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS)):
        out, _, _ = gpu_step(inp, part, mode)
        assert (out[0] == 0).all() and (out[2] == 0).all()
        _check_out(out, want, "bf16", f"P={part} mode={mode}")


def test_device_errors_are_reported_not_followed():
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 3, 20, 60)
    inp = wl.make_decode_inputs(cfg, seed=9)
    d = _to(inp, "cuda")
    kc, vc = d["key_cache"].clone(), d["value_cache"].clone()
    pa.pa_device_status(clear=True)
    # a slot past the cache is skipped and flagged
    sm = d["slot_mapping"].clone()
    sm[1] = inp.num_blocks * cfg.block_size + 5
    before = kc.clone()
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], kc, vc, sm)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_SLOT
    changed = (wl.raw_view(kc, "bf16") != wl.raw_view(before, "bf16")).flatten(1).any(1)
    assert changed.sum() <= 2          # only the two valid tokens' blocks
    # a block id past the cache reads zeros and is flagged
    out = torch.empty_like(d["q"])
    bt = d["block_tables"].clone()
    bt[0, 0] = inp.num_blocks + 3
    pa.pa_decode(out, d["q"], kc, vc, bt, d["context_lens"], inp.max_ctx, inp.scale)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_BLOCK
    # a context length beyond max_ctx is clamped and flagged
    cl = d["context_lens"].clone()
    cl[2] = inp.max_ctx + 100
    ws = torch.empty(pa.pa_decode_workspace_size(3, 32, 128, inp.max_ctx, 16), dtype=torch.uint8,
                     device="cuda")
    pa.pa_decode(out, d["q"], kc, vc, d["block_tables"], cl, inp.max_ctx, inp.scale,
                 partition=16, workspace=ws)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_CONTEXT
    assert pa.pa_device_status() == 0


@pytest.mark.parametrize("nseq,lo,hi", [(1, 1, 3), (3, 1, 40), (40, 1, 400), (7, 900, 3000)])
def test_balanced_grid_cuts(nseq, lo, hi):
    """Persistent balanced decode: fewer blocks than CTAs, items cut across many
    CTAs, and many small items per CTA all match the oracle."""
    cfg = wl.DecodeConfig("bal", nseq, 16, 4, 128, 16, "bf16", "bf16", lo, hi)
    inp = wl.make_decode_inputs(cfg, seed=nseq * 31 + hi)
    want, _, _ = oracle_step(inp)
    for mode in BOTH:
        out, _, _ = gpu_step(inp, -1, mode)
        _check_out(out, want, "bf16", f"mode={mode}")
    assert pa.pa_device_status() == 0


def test_balanced_many_pieces_per_cta():
    """Hundreds of short sequences: each persistent CTA walks tens of pieces,
    wrapping its descriptor ring several times."""
    cfg = wl.DecodeConfig("ringwrap", 512, 32, 8, 128, 16, "bf16", "bf16", 1, 48)
    inp = wl.make_decode_inputs(cfg, seed=5)
    want, _, _ = oracle_step(inp)
    pa.pa_device_status(clear=True)
    for mode in BOTH:
        out, _, _ = gpu_step(inp, -1, mode)
        bits = pa.pa_device_status()
        assert bits == 0, f"device status {bits:#x} (mode {mode})"
        _check_out(out, want, "bf16", f"mode={mode}")


HEAD_GROUPS = [(bs, G, D, dt, hkv) for bs in (8, 16, 32) for G in (2, 4, 16) for D in (64, 128)
               for dt in ("bf16", "f16", "fp8_e4m3") for hkv in (4, 8)
               if not (dt == "fp8_e4m3" and D == 64) and not (G == 16 and hkv == 8)]


@pytest.mark.parametrize("bs,G,D,dt,hkv", HEAD_GROUPS)
def test_head_groups(bs, G, D, dt, hkv):
    """Four kv heads per CTA (one per consumer warp, one tensor-map copy per
    block for all four) against the oracle, single pass and split-K, paired
    8-token blocks included; and against one head per CTA."""
    qdt = dt if dt != "fp8_e4m3" else "bf16"
    cfg = wl.DecodeConfig(f"hg_{bs}_{G}_{D}_{dt}_{hkv}", 5, hkv * G, hkv, D, bs, dt, qdt, 1,
                          9 * bs + 3, fp8_scaled=dt == "fp8_e4m3")
    inp = wl.make_decode_inputs(cfg, seed=bs * 7 + G * 3 + D + hkv)
    want, _, _ = oracle_step(inp)
    for part in (0, 2 * bs, 64):
        for mode in (pa.DECODE_DEFAULT, pa.DECODE_DEFAULT | pa.DECODE_ONE_HEAD_PER_CTA):
            out, _, _ = gpu_step(inp, part, mode)
            _check_out(out, want, dt, f"P={part} mode={mode}")
    assert pa.pa_device_status() == 0
