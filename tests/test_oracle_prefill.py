"""Pins for the oracle's paged prefill / chunked-prefill attention.

"01. PagedAttention 详解" §4, prefill: the new tokens' K and V are written
through the block table, then ordinary (causal, decoder) attention runs over the
cache.  The oracle is checked against things other than itself:
* torch's scaled_dot_product_attention in float64 with an explicit boolean
  causal mask offset by the cached length, on K/V gathered with torch indexing
  (catches a wrong position offset, an off-by-one in the causal bound, a wrong
  kv-head mapping, a dropped scale);
* a chunk of one token is a decode step: equal to the decode oracle's row;
* chunk invariance: a token's row does not depend on how the prompt was cut
  into chunks (one call over the whole prompt = the last chunk alone);
* causality: K/V past a row's position never change it, one at or before it
  does;
* closed form: the first token of a prefill from an empty cache returns v_0.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl


def _after_append(inp: wl.PrefillInputs):
    cfg = inp.cfg
    k, v = oracle.reshape_and_cache(inp.key_new, inp.value_new, cfg.dtype, inp.key_cache,
                                    inp.value_cache, cfg.dtype, inp.slot_mapping,
                                    cfg.block_size)
    kc = torch.from_numpy(k).view(inp.key_cache.dtype).reshape(inp.key_cache.shape)
    vc = torch.from_numpy(v).view(inp.value_cache.dtype).reshape(inp.value_cache.shape)
    return kc, vc


def _prefill(inp, kc, vc, q=None, qs=None, lens=None, rows=None):
    cfg = inp.cfg
    return oracle.paged_prefill(inp.q if q is None else q, cfg.dtype, kc, vc, cfg.dtype,
                                inp.block_tables, inp.context_lens if lens is None else lens,
                                inp.query_start if qs is None else qs, inp.scale, rows=rows)


def _sdpa_reference(inp: wl.PrefillInputs, kc, vc) -> np.ndarray:
    cfg = inp.cfg
    bs, G = cfg.block_size, cfg.group
    kf, vf, qf = kc.to(torch.float64), vc.to(torch.float64), inp.q.to(torch.float64)
    outs = []
    for s in range(cfg.num_seqs):
        a, b = int(inp.query_start[s]), int(inp.query_start[s + 1])
        n = int(inp.context_lens[s])
        L = b - a
        pos = torch.arange(n)
        blk = inp.block_tables[s].long()[pos // bs]
        K = kf[blk, pos % bs].permute(1, 0, 2).repeat_interleave(G, dim=0)   # [Hq, n, D]
        V = vf[blk, pos % bs].permute(1, 0, 2).repeat_interleave(G, dim=0)
        Q = qf[a:b].permute(1, 0, 2)                                         # [Hq, L, D]
        qpos = torch.arange(n - L, n)[:, None]
        mask = torch.arange(n)[None, :] <= qpos                              # [L, n]
        o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                             scale=inp.scale)
        outs.append(o.permute(1, 0, 2))
    return torch.cat(outs).numpy()


CASES = [
    wl.PrefillConfig("mha_chunks", 3, 4, 4, 64, 16, "bf16", 1, 40, 0, 50),
    wl.PrefillConfig("gqa4_bs8", 3, 8, 2, 64, 8, "f16", 5, 30, 0, 20),
    wl.PrefillConfig("gqa8_bs32_d128", 2, 16, 2, 128, 32, "bf16", 10, 70, 30, 90),
    wl.PrefillConfig("from_empty", 2, 8, 2, 64, 16, "bf16", 20, 50, 0, 0),
    wl.PrefillConfig("g16", 2, 16, 1, 64, 16, "f16", 3, 9, 0, 33),
]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_prefill_matches_masked_sdpa_on_the_unpaged_gather(cfg):
    inp = wl.make_prefill_inputs(cfg, seed=11)
    kc, vc = _after_append(inp)
    got = _prefill(inp, kc, vc)
    want = _sdpa_reference(inp, kc, vc)
    assert got.shape == want.shape
    assert np.abs(got - want).max() < 1e-12


def test_single_token_chunk_is_the_decode_step():
    cfg = wl.PrefillConfig("decode_like", 4, 8, 2, 64, 16, "bf16", 1, 1, 1, 100)
    inp = wl.make_prefill_inputs(cfg, seed=3)
    kc, vc = _after_append(inp)
    got = _prefill(inp, kc, vc)                               # T = S rows
    dec = oracle.paged_decode(inp.q, "bf16", kc, vc, "bf16", inp.block_tables,
                              inp.context_lens, inp.scale)
    assert np.array_equal(got, dec)


def test_rows_do_not_depend_on_the_chunking():
    # one prompt of 70 tokens from an empty cache ...
    cfg = wl.PrefillConfig("whole", 1, 8, 2, 64, 16, "bf16", 70, 70, 0, 0)
    inp = wl.make_prefill_inputs(cfg, seed=5)
    kc, vc = _after_append(inp)
    whole = _prefill(inp, kc, vc)
    # ... against its last 23 tokens as a chunk over 47 cached ones (same cache)
    last = 23
    q = inp.q[-last:].contiguous()
    qs = torch.tensor([0, last], dtype=torch.int32)
    chunk = _prefill(inp, kc, vc, q=q, qs=qs)
    assert np.array_equal(chunk, whole[-last:])
    # and sampled rows equal the full computation
    rows = [0, 5, 69]
    assert np.array_equal(_prefill(inp, kc, vc, rows=rows), whole[rows])


def test_causality():
    cfg = wl.PrefillConfig("causal", 1, 4, 4, 64, 16, "f16", 40, 40, 0, 0)
    inp = wl.make_prefill_inputs(cfg, seed=9)
    kc, vc = _after_append(inp)
    base = _prefill(inp, kc, vc)
    p = 17
    blk = int(inp.block_tables[0, (p + 1) // 16])
    k2, v2 = kc.clone(), vc.clone()
    k2[blk, (p + 1) % 16] += 1.0                              # a key after position p
    v2[blk, (p + 1) % 16] -= 2.0
    moved = _prefill(inp, k2, v2)
    assert np.array_equal(moved[: p + 1], base[: p + 1])
    assert not np.array_equal(moved[p + 1], base[p + 1])
    blk0 = int(inp.block_tables[0, p // 16])
    v3 = vc.clone()
    v3[blk0, p % 16] += 1.0                                   # the value at position p
    assert not np.array_equal(_prefill(inp, kc, v3)[p], base[p])


def test_first_token_of_a_prefill_returns_its_value():
    cfg = wl.PrefillConfig("first", 2, 8, 2, 64, 16, "bf16", 12, 12, 0, 0)
    inp = wl.make_prefill_inputs(cfg, seed=2)
    kc, vc = _after_append(inp)
    got = _prefill(inp, kc, vc)
    for s in range(2):
        row = int(inp.query_start[s])
        blk = int(inp.block_tables[s, 0])
        v0 = vc[blk, 0].to(torch.float64).numpy()              # [Hkv, D]
        want = np.repeat(v0, cfg.group, axis=0)
        assert np.array_equal(got[row], want)


def test_bad_chunk_lengths_are_rejected():
    cfg = wl.PrefillConfig("bad", 2, 4, 4, 64, 16, "bf16", 3, 3, 0, 5)
    inp = wl.make_prefill_inputs(cfg, seed=1)
    kc, vc = _after_append(inp)
    lens = inp.context_lens.clone()
    lens[0] = 2                                               # fewer tokens than the chunk
    with pytest.raises(oracle.OracleError):
        _prefill(inp, kc, vc, lens=lens)
