"""Pins for the oracle's paged decode attention, cache append and block copy.

The attention oracle is checked against things other than itself:
* torch's scaled_dot_product_attention in float64 on K/V gathered into
  contiguous tensors with torch indexing (a library routine on the unpaged
  data; catches a wrong gather index, a wrong kv-head mapping, a dropped scale);
* invariance under any relabelling of physical block ids, and identical outputs
  when sequences share prefix blocks instead of holding private copies
  ("01. PagedAttention 详解" §3: physical blocks need not be adjacent; §6: the
  same physical block may sit in several tables);
* softmax weights that are non-negative and sum to one;
* closed forms: one token gives its value row, q = 0 gives the mean of V, one
  logit far above the rest picks that value, GQA equals MHA with each kv head
  replicated over its group;
* poisoned storage (unused blocks, tail slots, table entries past the end) is
  never read; a NaN in an attended key or value reaches exactly the outputs
  that textbook attention (and SDPA) sends it to.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl


def _gather_sdpa(inp: wl.DecodeInputs, kc=None, vc=None, tables=None) -> np.ndarray:
    """Unpaged reference: torch indexing to gather, torch SDPA (float64) to attend."""
    cfg = inp.cfg
    kc = inp.key_cache if kc is None else kc
    vc = inp.value_cache if vc is None else vc
    tables = inp.block_tables if tables is None else tables
    kf = kc.to(torch.float64) * inp.k_scale
    vf = vc.to(torch.float64) * inp.v_scale
    qf = inp.q.to(torch.float64)
    bs, G = cfg.block_size, cfg.group
    outs = []
    for s in range(cfg.num_seqs):
        n = int(inp.context_lens[s])
        pos = torch.arange(n)
        blk = tables[s].long()[pos // bs]
        K = kf[blk, pos % bs]                        # [n, Hkv, D]
        V = vf[blk, pos % bs]
        K = K.permute(1, 0, 2).repeat_interleave(G, dim=0)   # [Hq, n, D]
        V = V.permute(1, 0, 2).repeat_interleave(G, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            qf[s][:, None, :], K, V, scale=inp.scale)[:, 0, :]
        outs.append(o)
    return torch.stack(outs).numpy()


def _oracle(inp: wl.DecodeInputs, kc=None, vc=None, tables=None, q=None, lens=None):
    cfg = inp.cfg
    return oracle.paged_decode(
        inp.q if q is None else q, cfg.q_dtype,
        inp.key_cache if kc is None else kc, inp.value_cache if vc is None else vc,
        cfg.kv_dtype, inp.block_tables if tables is None else tables,
        inp.context_lens if lens is None else lens, inp.scale, inp.k_scale, inp.v_scale)


def _torch_cache(raw: np.ndarray, like: torch.Tensor) -> torch.Tensor:
    t = torch.from_numpy(raw)
    return t.view(like.dtype).reshape(like.shape)


def _step_caches(inp: wl.DecodeInputs):
    cfg = inp.cfg
    kc, vc = inp.key_cache, inp.value_cache
    if inp.copy_pairs.numel():
        k2, v2 = oracle.copy_blocks(kc, vc, inp.copy_pairs)
        kc, vc = _torch_cache(k2, kc), _torch_cache(v2, vc)
    k3, v3 = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.q_dtype, kc, vc,
                                      cfg.kv_dtype, inp.slot_mapping, cfg.block_size,
                                      inp.k_scale, inp.v_scale)
    return _torch_cache(k3, kc), _torch_cache(v3, vc)


SMALL = [
    wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"],
    wl.small_variant(wl.DECODE_WORKLOADS["llama2_7b_mha_fp16_b64"], 3, 1, 70),
    wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 3, 1, 90),
    wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 3, 1, 70, prefix_tokens=64),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_oracle_matches_sdpa_on_unpaged_gather(cfg):
    inp = wl.make_decode_inputs(cfg, seed=11)
    kc, vc = _step_caches(inp)
    got = _oracle(inp, kc, vc)
    ref = _gather_sdpa(inp, kc, vc)
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bs,G,D", [(8, 1, 64), (16, 2, 64), (32, 4, 128), (8, 8, 128)])
def test_oracle_matches_sdpa_shapes(bs, G, D):
    cfg = wl.DecodeConfig("shape", 3, 2 * G, 2, D, bs, "bf16", "bf16", 1, 3 * bs + 1)
    inp = wl.make_decode_inputs(cfg, seed=bs * 100 + G)
    kc, vc = _step_caches(inp)
    np.testing.assert_allclose(_oracle(inp, kc, vc), _gather_sdpa(inp, kc, vc), rtol=0, atol=1e-12)


def test_block_id_relabelling_invariance():
    inp = wl.make_decode_inputs(wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 4, 20, 80), seed=5)
    kc, vc = _step_caches(inp)
    base = _oracle(inp, kc, vc)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(inp.num_blocks, generator=g)        # old id -> new id
    kc2, vc2 = torch.empty_like(kc), torch.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = inp.block_tables.clone()
    m = t2 >= 0
    t2[m] = perm[t2[m].long()].to(torch.int32)
    again = _oracle(inp, kc2, vc2, t2)
    assert np.array_equal(base, again)


def test_shared_prefix_equals_private_copies():
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 4, 5, 60, prefix_tokens=96)
    inp = wl.make_decode_inputs(cfg, seed=8)
    kc, vc = _step_caches(inp)
    shared = _oracle(inp, kc, vc)
    # give every sequence but the first its own copy of the prefix blocks
    nb = inp.num_blocks
    npre = cfg.prefix_tokens // cfg.block_size
    pre = inp.block_tables[0, :npre].long()
    extra = (cfg.num_seqs - 1) * npre
    kc2 = torch.cat([kc, torch.empty((extra,) + tuple(kc.shape[1:]), dtype=kc.dtype)])
    vc2 = torch.cat([vc, torch.empty((extra,) + tuple(vc.shape[1:]), dtype=vc.dtype)])
    t2 = inp.block_tables.clone()
    for s in range(1, cfg.num_seqs):
        ids = torch.arange(nb + (s - 1) * npre, nb + s * npre)
        kc2[ids] = kc[pre]
        vc2[ids] = vc[pre]
        t2[s, :npre] = ids.to(torch.int32)
    private = _oracle(inp, kc2, vc2, t2)
    assert np.array_equal(shared, private)


def test_weights_sum_to_one():
    inp = wl.make_decode_inputs(wl.small_variant(wl.DECODE_WORKLOADS["llama3_8b_gqa_bf16_b128"], 3, 1, 200), seed=2)
    kc, vc = _step_caches(inp)
    for s in range(3):
        for h in (0, 5, 31):
            w = oracle.decode_weights(inp.q, "bf16", kc, "bf16", inp.block_tables,
                                      inp.context_lens, inp.scale, s, h)
            assert w.size == int(inp.context_lens[s])
            assert (w >= 0).all()
            assert abs(w.sum() - 1.0) < 1e-12


def _single(cfg_kw, seed=0):
    cfg = wl.DecodeConfig("special", 1, 4, 2, 64, 16, "f32", "f32", 0, 0, **cfg_kw)
    return wl.make_decode_inputs(cfg, seed)


def test_one_token_gives_its_value_row():
    inp = _single(dict(fixed_lens=(1,)))
    kc, vc = _step_caches(inp)
    out = _oracle(inp, kc, vc)
    b = int(inp.block_tables[0, 0])
    v0 = vc[b, 0].to(torch.float64).numpy()            # [Hkv, D]
    np.testing.assert_array_equal(out[0], np.repeat(v0, 2, axis=0))


def test_zero_query_gives_mean_of_values():
    inp = _single(dict(fixed_lens=(37,)))
    kc, vc = _step_caches(inp)
    q0 = torch.zeros_like(inp.q)
    out = _oracle(inp, kc, vc, q=q0)
    blk = inp.block_tables[0].long()[torch.arange(37) // 16]
    V = vc[blk, torch.arange(37) % 16].to(torch.float64)  # [37, Hkv, D]
    mean = V.mean(0).numpy()
    np.testing.assert_allclose(out[0], np.repeat(mean, 2, axis=0), rtol=0, atol=1e-13)


def test_dominant_logit_selects_its_value():
    inp = _single(dict(fixed_lens=(40,)))
    kc, vc = _step_caches(inp)
    kc = kc.clone()
    q = torch.zeros_like(inp.q)
    q[0, :, 0] = 1.0
    # token 23 gets a key whose first coordinate is 8000 above every other key's
    b, o = int(inp.block_tables[0, 1]), 23 % 16
    kc[b, o, :, 0] = 8000.0 / inp.scale
    out = _oracle(inp, kc, vc, q=q)
    np.testing.assert_array_equal(out[0], np.repeat(vc[b, o].to(torch.float64).numpy(), 2, axis=0))


def test_gqa_equals_replicated_mha():
    cfg = wl.DecodeConfig("gqa", 3, 8, 2, 64, 16, "f16", "f16", 1, 50)
    inp = wl.make_decode_inputs(cfg, seed=4)
    kc, vc = _step_caches(inp)
    gqa = _oracle(inp, kc, vc)
    kc4 = kc.repeat_interleave(4, dim=2)
    vc4 = vc.repeat_interleave(4, dim=2)
    mha = oracle.paged_decode(inp.q, "f16", kc4, vc4, "f16", inp.block_tables,
                              inp.context_lens, inp.scale)
    assert np.array_equal(gqa, mha)


def test_poison_is_never_read():
    # the generator fills unused blocks / tails with NaN and pads tables with -1
    inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"], seed=0)
    assert torch.isnan(inp.key_cache[inp.free_blocks.long()]).all()
    assert (inp.block_tables == -1).any()
    kc, vc = _step_caches(inp)
    assert np.isfinite(_oracle(inp, kc, vc)).all()


def test_nan_reaches_exactly_the_attending_outputs():
    """A NaN in an attended key makes the whole output row of each query head of
    that kv head NaN; a NaN in one dimension of an attended value makes only
    that output dimension NaN; the same NaN past the length reaches nothing.
    torch SDPA (float64) on the unpaged gather agrees element for element, and
    every untouched output equals the clean run's exactly."""
    cfg = wl.DecodeConfig("nan", 3, 8, 2, 64, 16, "f32", "f32", 20, 60)
    inp = wl.make_decode_inputs(cfg, seed=4)
    kc, vc = _step_caches(inp)
    clean = _oracle(inp, kc, vc)
    G, bs = cfg.group, cfg.block_size
    kp, vp = kc.clone(), vc.clone()
    n0, n2 = int(inp.context_lens[0]), int(inp.context_lens[2])
    b, o = int(inp.block_tables[0, 7 // bs]), 7 % bs
    kp[b, o, 1, 3] = float("nan")                      # key of token 7, sequence 0, kv head 1
    b, o = int(inp.block_tables[2, (n2 - 1) // bs]), (n2 - 1) % bs
    vp[b, o, 0, 5] = float("nan")                      # value dim 5 of the last token of seq 2
    if n0 % bs:                                         # the slot after sequence 0's last token
        b, o = int(inp.block_tables[0, n0 // bs]), n0 % bs
        kp[b, o, 0, :] = float("nan")
        vp[b, o, 0, :] = float("nan")
    got = _oracle(inp, kp, vp)
    want = np.zeros_like(got, dtype=bool)
    want[0, G:2 * G, :] = True
    want[2, :G, 5] = True
    assert np.array_equal(np.isnan(got), want)
    assert np.array_equal(got[~want], clean[~want])
    ref = _gather_sdpa(inp, kp, vp)
    assert np.array_equal(np.isnan(ref), want)
    assert np.abs(ref[~want] - got[~want]).max() < 1e-12


def test_zero_length_sequence_gives_zero_row():
    cfg = wl.DecodeConfig("empty", 2, 4, 4, 64, 16, "f32", "f32", 0, 0, fixed_lens=(0, 5))
    inp = wl.make_decode_inputs(cfg, seed=1)
    kc, vc = _step_caches(inp)
    out = _oracle(inp, kc, vc)
    assert (out[0] == 0).all()
    assert np.isfinite(out[1]).all()


def test_bad_block_id_is_an_error():
    inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"], seed=0)
    t = inp.block_tables.clone()
    t[0, 0] = inp.num_blocks
    with pytest.raises(oracle.OracleError):
        _oracle(inp, tables=t)


# ---------------------------------------------------------------- append / copy

@pytest.mark.parametrize("name", ["tiny_paged_decode_fp32", "llama2_7b_mha_fp16_b64",
                                  "llama3_8b_gqa_bf16_b128"])
def test_append_places_rows_by_slot(name):
    base = wl.DECODE_WORKLOADS[name]
    cfg = base if base.fixed_lens else wl.small_variant(base, 5, 1, 70)
    inp = wl.make_decode_inputs(cfg, seed=3)
    kc, vc = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.q_dtype, inp.key_cache,
                                      inp.value_cache, cfg.kv_dtype, inp.slot_mapping,
                                      cfg.block_size)
    ek = oracle.raw(inp.key_cache).copy()
    ev = oracle.raw(inp.value_cache).copy()
    for t, slot in enumerate(inp.slot_mapping.tolist()):
        ek[slot // cfg.block_size, slot % cfg.block_size] = oracle.raw(inp.key_new)[t]
        ev[slot // cfg.block_size, slot % cfg.block_size] = oracle.raw(inp.value_new)[t]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_append_fp8_matches_torch_quantisation_and_skips_negative_slots():
    cfg = wl.small_variant(wl.DECODE_WORKLOADS["prefix_shared_fp8_b256"], 6, 1, 40, prefix_tokens=32)
    inp = wl.make_decode_inputs(cfg, seed=6)
    sm = inp.slot_mapping.clone()
    sm[2] = -1
    kc, vc = oracle.reshape_and_cache(inp.key_new, inp.value_new, "bf16", inp.key_cache,
                                      inp.value_cache, "fp8_e4m3", sm, cfg.block_size,
                                      inp.k_scale, inp.v_scale)
    ek = oracle.raw(inp.key_cache).copy()
    for t, slot in enumerate(sm.tolist()):
        if slot < 0:
            continue
        y = (inp.key_new[t].float() / torch.tensor(inp.k_scale, dtype=torch.float32))
        y = y.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        ek[slot // cfg.block_size, slot % cfg.block_size] = y
    assert np.array_equal(kc, ek)


def test_append_out_of_range_slot_is_an_error():
    inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"], seed=0)
    sm = inp.slot_mapping.clone()
    sm[1] = inp.num_blocks * 16
    with pytest.raises(oracle.OracleError):
        oracle.reshape_and_cache(inp.key_new, inp.value_new, "f32", inp.key_cache,
                                 inp.value_cache, "f32", sm, 16)


def test_copy_blocks_and_rejections():
    inp = wl.make_decode_inputs(wl.DECODE_WORKLOADS["tiny_paged_decode_fp32"], seed=0)
    pairs = torch.tensor([[3, 10], [5, 11], [3, 12]], dtype=torch.int32)
    kc, vc = oracle.copy_blocks(inp.key_cache, inp.value_cache, pairs)
    ek, ev = oracle.raw(inp.key_cache).copy(), oracle.raw(inp.value_cache).copy()
    for s, d in pairs.tolist():
        ek[d] = ek[s]
        ev[d] = ev[s]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)
    for bad in ([[1, 2], [3, 2]], [[1, 2], [2, 4]], [[1, 24]], [[-1, 3]]):
        with pytest.raises(oracle.OracleError):
            oracle.copy_blocks(inp.key_cache, inp.value_cache, torch.tensor(bad, dtype=torch.int32))
