"""NaN propagation on every decode and prefill path, against the fp64 oracle.

The oracle is textbook softmax attention: a NaN in the key of a token a query
attends to makes that query's weights, and so its whole output row, NaN; a NaN
in one dimension of a value makes that dimension of the output NaN and leaves
the others alone; a NaN in a slot past a sequence's length (or, in prefill,
past a query's causal bound) reaches nothing.  The kernels must agree: the NaN
pattern of the output equals the oracle's element for element, and the finite
elements meet the usual bars.  An empty row is zero (its sum is exactly 0), so
the output's normalisation must tell an empty row from a NaN sum -- a test on
"sum > 0" would turn the NaN rows into zero rows.

Cases: one-pass, split-K, balanced and grouped-partition decode with both
consumers and with one kv head per CTA; fp8 and MHA caches; the shared-prefix
decode with a NaN in the shared prefix (every sequence's row of that head) or
in one sequence's suffix, per-CTA and persistent suffix passes; prefill with a
NaN in a cached token and in a new token (rows from that position on).
"""
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
    pa.pa_decode_select(pa.DECODE_DEFAULT)


def _stepped(inp: wl.DecodeInputs):
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
    return (torch.from_numpy(k3).view(kc.dtype).reshape(kc.shape).clone(),
            torch.from_numpy(v3).view(vc.dtype).reshape(vc.shape).clone())


def _poison(cache, tables, bs, s, t, g, d=None):
    """NaN into token t of sequence s, kv head g (every dim, or dim d)."""
    b, o = int(tables[s, t // bs]), t % bs
    if d is None:
        cache[b, o, g, :] = float("nan")
    else:
        cache[b, o, g, d] = float("nan")


def _compare(got: torch.Tensor, want: np.ndarray, tol: float, what: str, expect_nan: bool = True):
    g = got.to(torch.float64).numpy()
    ng, nw = np.isnan(g), np.isnan(want)
    assert nw.any() == expect_nan, f"{what}: the case must (not) put NaN in the oracle's output"
    bad = np.argwhere(ng != nw)
    assert bad.size == 0, f"{what}: NaN pattern differs at {bad[:4].tolist()} ({len(bad)} elements)"
    assert np.isfinite(g[~ng]).all(), f"{what}: infinite output"
    err = np.abs(g[~ng] - want[~nw]).max()
    assert err <= tol, f"{what}: max abs error {err:.3g} on the finite elements"


def _decode(inp, kc, vc, partition, mode):
    cfg = inp.cfg
    q, bt, cl = inp.q.cuda(), inp.block_tables.cuda(), inp.context_lens.cuda()
    S, Hq, D = q.shape
    nb = pa.pa_decode_workspace_size(S, Hq, D, inp.max_ctx, partition)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, 7.0)
    pa.pa_decode_select(mode)
    pa.pa_decode(out, q, kc.cuda(), vc.cuda(), bt, cl, inp.max_ctx, inp.scale, inp.k_scale,
                 inp.v_scale, partition, ws if nb else None)
    torch.cuda.synchronize()
    pa.pa_decode_select(pa.DECODE_DEFAULT)
    return out.cpu()


def _oracle_decode(inp, kc, vc):
    cfg = inp.cfg
    return oracle.paged_decode(inp.q, cfg.q_dtype, kc, vc, cfg.kv_dtype, inp.block_tables,
                               inp.context_lens, inp.scale, inp.k_scale, inp.v_scale)


DECODE = [
    ("gqa_bf16", wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 5, 100, 700)),
    ("mha_f16", wl.small_variant(wl.DECODE_WORKLOADS["llama2_7b_mha_fp16_b64"], 3, 100, 500)),
    ("gqa_fp8", wl.DecodeConfig("nan_fp8", 4, 32, 8, 128, 32, "fp8_e4m3", "bf16", 100, 600,
                                cow_last_block=True, fp8_scaled=True)),
]
DECODE_MODES = {"auto": pa.DECODE_DEFAULT, "simt": pa.DECODE_DEFAULT | pa.DECODE_SIMT_ONLY,
                "grouped": pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS,
                "one_head": pa.DECODE_DEFAULT | pa.DECODE_ONE_HEAD_PER_CTA}


@pytest.mark.parametrize("name,cfg", DECODE, ids=[n for n, _ in DECODE])
@pytest.mark.parametrize("part_blocks", [0, 2, 7, -1], ids=["single", "p2", "p7", "balanced"])
def test_decode_nan(name, cfg, part_blocks):
    inp = wl.make_decode_inputs(cfg, seed=77)
    kc, vc = _stepped(inp)
    lens = inp.context_lens
    bs, G = cfg.block_size, cfg.num_q_heads // cfg.num_kv_heads
    s0 = int(lens.argmax())
    s1 = (s0 + 1) % cfg.num_seqs
    _poison(kc, inp.block_tables, bs, s0, int(lens[s0]) // 3, 1)            # a key, mid-sequence
    _poison(vc, inp.block_tables, bs, s1, int(lens[s1]) - 1, 0, d=5)        # a value dim, last token
    want = _oracle_decode(inp, kc, vc)
    # what the oracle says, spelled out: head group 1 of s0 NaN everywhere,
    # head group 0 of s1 NaN in dim 5 only, nothing else
    nan = np.isnan(want)
    assert nan[s0, G:2 * G].all() and nan[s1, :G, 5].all()
    assert nan.sum() == G * cfg.head_dim + G
    part = -1 if part_blocks < 0 else part_blocks * bs
    for mode_name, mode in DECODE_MODES.items():
        got = _decode(inp, kc, vc, part, mode)
        _compare(got, want, TOL[cfg.kv_dtype], f"{name} P={part_blocks} {mode_name}")
    assert pa.pa_device_status() == 0


def test_decode_nan_past_the_length_reaches_nothing():
    """The slot right after each sequence's last token (inside its last block)
    holds NaN: no output changes."""
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 6, 1, 300)
    inp = wl.make_decode_inputs(cfg, seed=78)
    kc, vc = _stepped(inp)
    bs = cfg.block_size
    for s in range(cfg.num_seqs):
        n = int(inp.context_lens[s])
        if n % bs:                                   # room left in the last block
            for g in range(cfg.num_kv_heads):
                _poison(kc, inp.block_tables, bs, s, n, g)
                _poison(vc, inp.block_tables, bs, s, n, g)
    want = _oracle_decode(inp, kc, vc)
    for part in (0, 2 * bs, -1):
        for mode_name, mode in DECODE_MODES.items():
            got = _decode(inp, kc, vc, part, mode)
            _compare(got, want, TOL["bf16"], f"tail P={part} {mode_name}", expect_nan=False)


def test_long_split_decode_nan():
    """Grouped split-K partitions over thousands of tokens, NaN in one
    partition of one sequence."""
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["long_context_splitk_bf16_4x100k"], 2, 1500, 2100)
    inp = wl.make_decode_inputs(cfg, seed=79)
    kc, vc = _stepped(inp)
    _poison(kc, inp.block_tables, cfg.block_size, 1, 1234, 3)
    want = _oracle_decode(inp, kc, vc)
    for part in (0, 512):
        for mode in (pa.DECODE_DEFAULT, pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS):
            _compare(_decode(inp, kc, vc, part, mode), want, TOL["bf16"], f"P={part} mode={mode}")


SUFFIX_MODES = {"per_cta": pa.DECODE_DEFAULT,
                "persistent": pa.DECODE_DEFAULT | pa.DECODE_SUFFIX_PERSISTENT}


@pytest.mark.parametrize("where", ["prefix", "suffix"])
@pytest.mark.parametrize("suffix_hi", [300, 5000], ids=["fused", "split"])
def test_shared_prefix_nan(where, suffix_hi):
    base = wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"]
    nseq = 8 if suffix_hi < 4096 else 3
    cfg = wl.small_variant(base, nseq, 30 if suffix_hi < 4096 else 4200, suffix_hi,
                           prefix_tokens=256)
    inp = wl.make_decode_inputs(cfg, seed=80)
    kc, vc = _stepped(inp)
    G = cfg.num_q_heads // cfg.num_kv_heads
    if where == "prefix":      # the shared blocks: every sequence's rows of head group 2
        _poison(kc, inp.block_tables, cfg.block_size, 0, 100, 2)
    else:                      # one sequence's own suffix
        _poison(kc, inp.block_tables, cfg.block_size, 1, 256 + 10, 2)
    want = _oracle_decode(inp, kc, vc)
    nan = np.isnan(want)
    rows = nan.any(axis=(1, 2)).sum()
    assert rows == (nseq if where == "prefix" else 1) and nan[1, 2 * G:3 * G].all()
    q, bt, cl = inp.q.cuda(), inp.block_tables.cuda(), inp.context_lens.cuda()
    S, Hq, D = q.shape
    nb = pa.pa_decode_shared_prefix_workspace_size(S, Hq, cfg.num_kv_heads, D, cfg.block_size,
                                                   inp.max_ctx, 256, kc.dtype)
    ws = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
    kcd, vcd = kc.cuda(), vc.cuda()
    for mode_name, mode in SUFFIX_MODES.items():
        pa.pa_decode_select(mode)
        out = torch.full_like(q, 7.0)
        pa.pa_decode_shared_prefix(out, q, kcd, vcd, bt, cl, inp.max_ctx, inp.scale, 256,
                                   ws if nb else None, inp.k_scale, inp.v_scale)
        torch.cuda.synchronize()
        pa.pa_decode_select(pa.DECODE_DEFAULT)
        _compare(out.cpu(), want, TOL["fp8_e4m3"], f"{where} {mode_name}")
    assert pa.pa_device_status() == 0


PREFILL_KERNELS = {"single": pa.DECODE_DEFAULT,
                   "pair": pa.DECODE_DEFAULT | pa.PREFILL_CTA_PAIRS}


@pytest.mark.parametrize("kernel", sorted(PREFILL_KERNELS))
def test_prefill_nan(kernel):
    """A NaN key in a cached token reaches every new row of its head group; a
    NaN key in new token i reaches the rows at positions from i on (causal)."""
    cfg = wl.PrefillConfig("nan", 2, 8, 2, 128, 16, "bf16", 150, 300, 40, 200)
    inp = wl.make_prefill_inputs(cfg, seed=81)
    key_new = inp.key_new.clone()
    qs = inp.query_start
    c0 = int(inp.cached_lens[0])
    i1 = 37                                          # new token 37 of sequence 1, kv head 0
    key_new[int(qs[1]) + i1, 0, :] = float("nan")
    kc = inp.key_cache.clone()
    _poison(kc, inp.block_tables, cfg.block_size, 0, c0 // 2, 1)   # cached token of sequence 0
    k, v = oracle.reshape_and_cache(key_new, inp.value_new, cfg.dtype, kc, inp.value_cache,
                                    cfg.dtype, inp.slot_mapping, cfg.block_size)
    kco = torch.from_numpy(k).view(kc.dtype).reshape(kc.shape)
    vco = torch.from_numpy(v).view(kc.dtype).reshape(kc.shape)
    want = oracle.paged_prefill(inp.q, cfg.dtype, kco, vco, cfg.dtype, inp.block_tables,
                                inp.context_lens, inp.query_start, inp.scale)
    nan = np.isnan(want)
    L0, L1 = int(qs[1] - qs[0]), int(qs[2] - qs[1])
    G = cfg.num_q_heads // cfg.num_kv_heads
    assert nan[:L0, G:2 * G].all() and not nan[:L0, :G].any()
    assert nan[int(qs[1]) + i1:int(qs[2]), :G].all() and not nan[int(qs[1]):int(qs[1]) + i1].any()
    d = {k_: getattr(inp, k_).cuda() for k_ in ("q", "value_new", "slot_mapping", "block_tables",
                                                "context_lens", "query_start", "value_cache")}
    kcd = kc.cuda()
    vcd = d["value_cache"].clone()
    pa.pa_reshape_and_cache(key_new.cuda(), d["value_new"], kcd, vcd, d["slot_mapping"])
    out = torch.full_like(d["q"], 7.0)
    pa.pa_decode_select(PREFILL_KERNELS[kernel])
    pa.pa_prefill(out, d["q"], kcd, vcd, d["block_tables"], d["context_lens"], d["query_start"],
                  inp.max_query_len, inp.scale)
    torch.cuda.synchronize()
    pa.pa_decode_select(pa.DECODE_DEFAULT)
    assert pa.pa_device_status() == 0
    _compare(out.cpu(), want, TOL["bf16"], f"prefill {kernel} (L {L0}, {L1})")
