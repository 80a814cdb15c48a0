"""GPU parity of the shared-prefix (cascade) decode against the fp64 decode
oracle, through the C ABI.

pa_decode_shared_prefix must compute what pa_decode computes: the oracle is the
same textbook attention over each sequence's own gather.  Cases: fp8 and bf16
caches, prefixes of one chunk, several chunks and an uneven length; a sequence
whose table does not start with row 0's prefix blocks (its own prefix has other
values: a wrong fall-back shows up as an error), a sequence shorter than the
prefix and one that holds exactly the prefix.  Tolerances are the decode bars.

Short suffixes are decoded two ways, both checked: one CTA per (sequence, kv
head) suffix (the default) and the persistent grid (DECODE_SUFFIX_PERSISTENT:
groups of one CTA per kv head, each group streaming a run of whole sequences'
suffixes and folding the prefix records into each).  A batch of many short
suffixes puts several items on every CTA of the persistent grid.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_338_b200 as pa
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2, "fp8_e4m3": 3e-2}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


MODES = {"per_cta": pa.DECODE_DEFAULT,
         "persistent": pa.DECODE_DEFAULT | pa.DECODE_SUFFIX_PERSISTENT}


@pytest.fixture(params=sorted(MODES))
def mode(request):
    pa.pa_decode_select(MODES[request.param])
    yield request.param
    pa.pa_decode_select(pa.DECODE_DEFAULT)


def _appended(inp: wl.DecodeInputs):
    """Host caches after the step's copy-on-write and append (the oracle's)."""
    cfg = inp.cfg
    kc, vc = inp.key_cache, inp.value_cache
    if inp.copy_pairs.numel():
        k2, v2 = oracle.copy_blocks(kc, vc, inp.copy_pairs)
        kc = torch.from_numpy(k2).view(kc.dtype).reshape(kc.shape)
        vc = torch.from_numpy(v2).view(vc.dtype).reshape(vc.shape)
    k3, v3 = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.q_dtype, kc, vc,
                                      cfg.kv_dtype, inp.slot_mapping, cfg.block_size,
                                      inp.k_scale, inp.v_scale)
    return (torch.from_numpy(k3).view(kc.dtype).reshape(kc.shape),
            torch.from_numpy(v3).view(vc.dtype).reshape(vc.shape))


def _run(inp, kc, vc, tables, lens, prefix_tokens, max_ctx):
    cfg = inp.cfg
    d = {k: v.cuda() for k, v in (("q", inp.q), ("kc", kc), ("vc", vc), ("bt", tables),
                                  ("cl", lens))}
    S, Hq, D = inp.q.shape
    nb = pa.pa_decode_shared_prefix_workspace_size(S, Hq, cfg.num_kv_heads, D, cfg.block_size,
                                                   max_ctx, prefix_tokens, d["kc"].dtype)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(d["q"], float("nan"))
    pa.pa_decode_shared_prefix(out, d["q"], d["kc"], d["vc"], d["bt"], d["cl"], max_ctx,
                               inp.scale, prefix_tokens, ws if nb else None, inp.k_scale,
                               inp.v_scale)
    torch.cuda.synchronize()
    return out.cpu()


def _check(got, inp, kc, vc, tables, lens, what):
    cfg = inp.cfg
    want = oracle.paged_decode(inp.q, cfg.q_dtype, kc, vc, cfg.kv_dtype, tables, lens, inp.scale,
                               inp.k_scale, inp.v_scale)
    g = got.to(torch.float64).numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want).max()
    assert err <= TOL[cfg.kv_dtype], f"{what}: max abs error {err:.3g}"


CASES = [
    # name, base config, seqs, suffix lo/hi, prefix tokens
    ("fp8_bs32_p256", wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 12, 1, 200, 256),
    ("fp8_bs32_p1024", wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 10, 30, 300, 1024),
    ("fp8_bs32_p96", wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 9, 1, 90, 96),
    ("bf16_bs16_p512", dataclasses.replace(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], kv_dtype="bf16", block_size=16,
                                           fp8_scaled=False), 11, 1, 300, 512),
    ("f16_mha_bs8_p128", dataclasses.replace(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], kv_dtype="f16", q_dtype="f16",
                                             num_kv_heads=32, block_size=8, fp8_scaled=False),
     5, 1, 60, 128),
    ("fp8_q_f16_g8", dataclasses.replace(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], q_dtype="f16", num_q_heads=16,
                                         num_kv_heads=2), 7, 1, 100, 256),
    ("bf16_d64_g2", dataclasses.replace(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], kv_dtype="bf16", head_dim=64,
                                        num_q_heads=8, num_kv_heads=4, block_size=16,
                                        fp8_scaled=False), 6, 1, 150, 256),
    # 1600 items of 1..4 blocks: several whole items per CTA of the persistent grid
    ("fp8_bs32_many", wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 200, 1, 120, 128),
]


@pytest.mark.parametrize("name,base,nseq,lo,hi,prefix", CASES, ids=[c[0] for c in CASES])
def test_shared_prefix_matches_decode(name, base, nseq, lo, hi, prefix, mode):
    cfg = wl.small_variant(base, nseq, lo, hi, prefix_tokens=prefix)
    inp = wl.make_decode_inputs(cfg, seed=len(name))
    kc, vc = _appended(inp)
    pa.pa_device_status(clear=True)
    out = _run(inp, kc, vc, inp.block_tables, inp.context_lens, prefix, inp.max_ctx)
    assert pa.pa_device_status() == 0
    _check(out, inp, kc, vc, inp.block_tables, inp.context_lens, name)


def test_sequences_outside_the_shared_prefix_fall_back(mode):
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 8, 20, 200, prefix_tokens=512)
    inp = wl.make_decode_inputs(cfg, seed=3)
    kc, vc = _appended(inp)
    tables, lens = inp.block_tables.clone(), inp.context_lens.clone()
    # sequence 1 starts with a block of its own, holding other values
    own = int(inp.free_blocks[0])
    g = torch.Generator().manual_seed(1)
    kc[own] = (torch.randn(kc[own].shape, generator=g) / inp.k_scale).clamp(-448, 448).to(kc.dtype)
    vc[own] = (torch.randn(vc[own].shape, generator=g) / inp.v_scale).clamp(-448, 448).to(vc.dtype)
    tables[1, 0] = own
    # sequence 2 holds fewer tokens than the prefix, sequence 3 exactly the prefix
    lens[2] = 300
    lens[3] = 512
    out = _run(inp, kc, vc, tables, lens, 512, inp.max_ctx)
    assert pa.pa_device_status() == 0
    _check(out, inp, kc, vc, tables, lens, "fall-back")


def test_prefix_longer_than_every_context_is_a_plain_decode():
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 4, 1, 30, prefix_tokens=64)
    inp = wl.make_decode_inputs(cfg, seed=8)
    kc, vc = _appended(inp)
    wide = torch.full((4, 8), -1, dtype=torch.int32)        # room for the declared prefix
    wide[:, :inp.block_tables.shape[1]] = inp.block_tables
    out = _run(inp, kc, vc, wide, inp.context_lens, 64 + 32 * 4, inp.max_ctx)
    assert pa.pa_device_status() == 0
    _check(out, inp, kc, vc, wide, inp.context_lens, "longer prefix")


def test_long_suffixes_take_the_split_path():
    """Suffixes past 4096 tokens are cut into 256-token partitions and merged by
    the split-K merge; an irregular sequence is exact there too."""
    cfg = wl.small_variant(dataclasses.replace(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], kv_dtype="bf16", block_size=16,
                                               fp8_scaled=False, cow_last_block=False),
                           3, 4000, 5200, prefix_tokens=256)
    inp = wl.make_decode_inputs(cfg, seed=12)
    kc, vc = _appended(inp)
    tables, lens = inp.block_tables.clone(), inp.context_lens.clone()
    lens[1] = 200                                            # shorter than the prefix
    out = _run(inp, kc, vc, tables, lens, 256, inp.max_ctx)
    assert pa.pa_device_status() == 0
    _check(out, inp, kc, vc, tables, lens, "split")


def test_irregular_sequences_inside_a_long_batch(mode):
    """Regular and irregular sequences side by side in the runs of whole items a
    persistent CTA streams: a foreign first block, one shorter than the prefix,
    one holding exactly the prefix (an item with no suffix block), next to
    regular ones."""
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 160, 1, 100,
                           prefix_tokens=128)
    inp = wl.make_decode_inputs(cfg, seed=21)
    kc, vc = _appended(inp)
    tables, lens = inp.block_tables.clone(), inp.context_lens.clone()
    g = torch.Generator().manual_seed(5)
    for s, fb in ((5, 0), (50, 1), (51, 2)):
        own = int(inp.free_blocks[fb])
        kc[own] = (torch.randn(kc[own].shape, generator=g) / inp.k_scale).clamp(-448, 448).to(kc.dtype)
        vc[own] = (torch.randn(vc[own].shape, generator=g) / inp.v_scale).clamp(-448, 448).to(vc.dtype)
        tables[s, fb] = own                         # its prefix differs in block fb
    lens[7] = 70                                    # shorter than the prefix
    lens[8] = 128                                   # exactly the prefix
    lens[9] = 129                                   # one suffix token
    out = _run(inp, kc, vc, tables, lens, 128, inp.max_ctx)
    assert pa.pa_device_status() == 0
    _check(out, inp, kc, vc, tables, lens, "irregular in a long batch")
