"""GPU parity of the tensor-core prefill / chunked-prefill path against the fp64
oracle, through the C ABI.

Each case runs the whole prefill step of "01. PagedAttention 详解" §4: append
the new tokens' K, V through slot_mapping (bit-exact against the oracle), then
pa_prefill (max abs error against the oracle's double result: bf16 1e-2,
f16 2e-3, the decode bars: P is rounded to the operand type and accumulated in
fp32 as there).  Unused blocks, tail slots and table padding are poisoned.
Head size 128 runs two kernels, both checked: one CTA per pair of query tiles
(the default) and a cluster of two CTAs per pair (PREFILL_CTA_PAIRS).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


KERNELS = {"single": pa.DECODE_DEFAULT, "pair": pa.DECODE_DEFAULT | pa.PREFILL_CTA_PAIRS}


@pytest.fixture(params=sorted(KERNELS))
def kernel(request):
    pa.pa_decode_select(KERNELS[request.param])
    yield request.param
    pa.pa_decode_select(pa.DECODE_DEFAULT)


def gpu_prefill(inp: wl.PrefillInputs, max_query_len=None, tables=None, lens=None):
    d = {k: getattr(inp, k).cuda() for k in ("q", "key_cache", "value_cache", "key_new",
                                              "value_new", "slot_mapping", "block_tables",
                                              "context_lens", "query_start")}
    kc, vc = d["key_cache"].clone(), d["value_cache"].clone()
    pa.pa_reshape_and_cache(d["key_new"], d["value_new"], kc, vc, d["slot_mapping"])
    out = torch.full_like(d["q"], float("nan"))
    pa.pa_prefill(out, d["q"], kc, vc, d["block_tables"] if tables is None else tables.cuda(),
                  d["context_lens"] if lens is None else lens.cuda(), d["query_start"],
                  inp.max_query_len if max_query_len is None else max_query_len, inp.scale)
    torch.cuda.synchronize()
    return out.cpu(), kc.cpu(), vc.cpu()


def oracle_prefill(inp: wl.PrefillInputs, rows=None):
    cfg = inp.cfg
    k, v = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.dtype, inp.key_cache,
                                    inp.value_cache, cfg.dtype, inp.slot_mapping,
                                    cfg.block_size)
    kc = torch.from_numpy(k).view(inp.key_cache.dtype).reshape(inp.key_cache.shape)
    vc = torch.from_numpy(v).view(inp.value_cache.dtype).reshape(inp.value_cache.shape)
    out = oracle.paged_prefill(inp.q, cfg.dtype, kc, vc, cfg.dtype, inp.block_tables,
                               inp.context_lens, inp.query_start, inp.scale, rows=rows)
    return out, kc, vc


def _check(got: torch.Tensor, want: np.ndarray, dt: str, what: str):
    g = got.to(torch.float64).numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want).max()
    assert err <= TOL[dt], f"{what}: max abs error {err:.3g} > {TOL[dt]}"
    return err


def _bits_equal(a, b, dt):
    return torch.equal(wl.raw_view(a.contiguous(), dt), wl.raw_view(b.contiguous(), dt))


def test_first_case_small(kernel):
    cfg = wl.PrefillConfig("first", 2, 8, 2, 128, 16, "bf16", 5, 150, 0, 200)
    inp = wl.make_prefill_inputs(cfg, seed=1)
    want, kc_o, vc_o = oracle_prefill(inp)
    out, kc, vc = gpu_prefill(inp)
    assert pa.pa_device_status() == 0
    assert _bits_equal(kc, kc_o, "bf16") and _bits_equal(vc, vc_o, "bf16")
    _check(out, want, "bf16", "first")


SHAPES = [(G, D, bs, dt) for G in (1, 2, 4, 8, 16) for D in (64, 128) for bs in (8, 16, 32)
          for dt in ("bf16", "f16") if (G + D // 64 + bs // 8 + (dt == "f16")) % 2 == 0] + \
         [(4, 128, 16, "bf16"), (4, 128, 16, "f16"), (8, 128, 16, "bf16"), (1, 64, 32, "f16")]


@pytest.mark.parametrize("G,D,bs,dt", SHAPES)
def test_prefill_shapes(G, D, bs, dt, kernel):
    Hkv = 2
    cfg = wl.PrefillConfig(f"s{G}_{D}_{bs}_{dt}", 3, G * Hkv, Hkv, D, bs, dt, 1, 300, 0, 400)
    inp = wl.make_prefill_inputs(cfg, seed=G * 100 + D + bs)
    want, kc_o, vc_o = oracle_prefill(inp)
    out, kc, vc = gpu_prefill(inp)
    assert pa.pa_device_status() == 0
    assert _bits_equal(kc, kc_o, dt) and _bits_equal(vc, vc_o, dt)
    _check(out, want, dt, cfg.name)


@pytest.mark.parametrize("G", [1, 4, 16])
def test_tile_edges(G, kernel):
    """Chunk lengths at the query-tile size +-1, cached lengths that put the last
    key at a key-tile edge +-1, a one-token chunk and a chunk from an empty cache."""
    TQ = 128 // G
    Ls = (1, TQ - 1, TQ, TQ + 1, 2 * TQ + 3, 5, 128, 40)
    cs = tuple(max(0, c) for c in (0, 129 - (TQ - 1), 128 - TQ, 0, 255 - (2 * TQ + 3), 251, 0, 1))
    cfg = wl.PrefillConfig("edges", len(Ls), 2 * G, 2, 128, 16, "bf16", 0, 0, 0, 0,
                           fixed_q=Ls, fixed_ctx=cs)
    inp = wl.make_prefill_inputs(cfg, seed=G)
    want, _, _ = oracle_prefill(inp)
    out, _, _ = gpu_prefill(inp)
    assert pa.pa_device_status() == 0
    _check(out, want, "bf16", f"G={G}")


def test_empty_chunks_and_a_larger_grid():
    """Sequences with no new tokens write nothing; a max_query_len above the
    longest chunk launches query tiles that exit at once."""
    cfg = wl.PrefillConfig("holes", 4, 8, 2, 64, 16, "f16", 0, 0, 0, 0,
                           fixed_q=(0, 37, 0, 5), fixed_ctx=(10, 3, 0, 90))
    inp = wl.make_prefill_inputs(cfg, seed=4)
    want, _, _ = oracle_prefill(inp)
    out, _, _ = gpu_prefill(inp, max_query_len=300)
    assert pa.pa_device_status() == 0
    _check(out, want, "f16", "holes")


def test_long_context_rows_sampled():
    """The chunked-prefill bench workload at full size: sampled rows against the
    oracle (first, last and random rows of every sequence)."""
    cfg = wl.PREFILL_CONFIGS["llama3_8b_gqa_bf16_chunked_prefill"]
    inp = wl.make_prefill_inputs(cfg, seed=2)
    out, _, _ = gpu_prefill(inp)
    assert pa.pa_device_status() == 0
    g = torch.Generator().manual_seed(0)
    rows = []
    qs = inp.query_start.tolist()
    for s in range(cfg.num_seqs):
        a, b = qs[s], qs[s + 1]
        rows += [a, b - 1] + torch.randint(a, b, (2,), generator=g).tolist()
    want, _, _ = oracle_prefill(inp, rows=rows)
    _check(out[rows], want, "bf16", "sampled rows")


def test_device_errors_are_reported(kernel):
    cfg = wl.PrefillConfig("errs", 2, 8, 2, 128, 16, "bf16", 20, 20, 30, 30)
    inp = wl.make_prefill_inputs(cfg, seed=6)
    pa.pa_device_status(clear=True)
    bt = inp.block_tables.clone()
    bt[0, 1] = inp.num_blocks + 5                 # a block id past the cache
    gpu_prefill(inp, tables=bt)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_BLOCK
    lens = inp.context_lens.clone()
    lens[1] = 10                                  # fewer cached tokens than the chunk
    gpu_prefill(inp, lens=lens)
    assert pa.pa_device_status() & pa.PA_DEV_BAD_CONTEXT
    out, _, _ = gpu_prefill(inp)                  # the context is still usable
    assert pa.pa_device_status() == 0
    want, _, _ = oracle_prefill(inp)
    _check(out, want, "bf16", "after errors")
