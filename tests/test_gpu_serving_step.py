"""GPU parity of the serving step the pages describe, driven by the host block
pool: every step the pool makes room for each sequence's new token (a fresh
block at a block boundary, a copy-on-write when the last block is shared),
packs all tables into one host buffer, and the GPU then copies the blocks,
appends the new k, v and attends ("01. PagedAttention 详解" §4: append, then
attend; §10: the tables go to the GPU as one packed tensor per step;
intelliparadigm PagedAttention article §3.3: maybe_copy_block).

The GPU side takes its slots, copy pairs, tables and lengths from the
library's pool (pa_pool_step); the oracle side replays the same calls on
oracle.pool_model.PoolModel and feeds ITS tables to oracle.copy_blocks,
oracle.reshape_and_cache and oracle.paged_decode.  Checked every step: the
pool's and the model's slots, pairs, tables and lengths are identical, both
caches are bit-identical, and pa_decode / pa_decode_shared_prefix are within
the decode tolerance of the oracle.

The batch exercises what the pool decides: sequences that grow across block
boundaries, a shared prefix (seq_share_prefix), a sampling fork whose parent
then writes into a shared last block (copy-on-write), a prefix-cache hit on
live blocks and one on a freed block revived from the free queue
(seq_match_prefix), and sequences that leave and join mid-run.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.pool_model as pm
import paged_kv_cache_338_b200 as pa

pytestmark = pytest.mark.gpu

TOL = {"bf16": 1e-2, "fp8_e4m3": 3e-2}
TDT = {"bf16": torch.bfloat16, "fp8_e4m3": torch.float8_e4m3fn}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    pa.pa_device_status(clear=True)
    yield


class Twin:
    """The library's pool and the oracle's model, driven call for call."""

    def __init__(self, nb, bs):
        self.pool = pa.BlockPool(nb, bs)
        self.model = pm.PoolModel(nb, bs)

    def both(self, name, *args):
        a = getattr(self.pool, name)(*args)
        b = getattr(self.model, name)(*args)
        assert a == b, f"{name}{args}: pool {a} vs model {b}"
        return a

    def fill(self, seq, ntok):
        for _ in range(ntok):
            self.both("seq_append", seq)


def _draw(shape, dtype_name, g, scale=1.0):
    x = torch.randn(shape, generator=g)
    if dtype_name == "fp8_e4m3":
        x = (x / scale).clamp(-448.0, 448.0)
    return x.to(TDT[dtype_name])


@pytest.mark.parametrize("kv_dtype,bs", [("bf16", 16), ("fp8_e4m3", 32)])
def test_pool_driven_steps_match_the_oracle(kv_dtype, bs):
    NB, Hq, Hkv, D, MB, steps = 160, 8, 2, 128, 12, 24
    q_dtype = "bf16"
    g = torch.Generator().manual_seed(bs)
    k_scale = v_scale = 1.0
    if kv_dtype == "fp8_e4m3":
        k_scale, v_scale = 3.5 / 448.0, 4.0 / 448.0
    scale = 1.0 / np.sqrt(D)
    # every block holds finite values: a wrong block id reads wrong numbers
    kc_h = _draw((NB, bs, Hkv, D), kv_dtype, g, k_scale)
    vc_h = _draw((NB, bs, Hkv, D), kv_dtype, g, v_scale)
    kc_d, vc_d = kc_h.cuda(), vc_h.cuda()
    k_o, v_o = oracle.raw(kc_h).copy(), oracle.raw(vc_h).copy()

    t = Twin(NB, bs)
    prefix_tokens = 3 * bs
    owner = t.both("seq_new")
    t.fill(owner, prefix_tokens)
    prefix = t.pool.seq_blocks(owner)
    assert prefix == t.model.seq_blocks(owner)
    hashes = [0x1000 + i for i in range(len(prefix))]
    for b, h in zip(prefix, hashes):
        assert t.both("cache_block", b, h)
    A = t.both("seq_new")
    t.both("seq_share_prefix", A, prefix, prefix_tokens)
    t.fill(A, bs // 2 + 1)                      # a part-filled private block
    B = t.both("seq_new")
    t.both("seq_share_prefix", B, prefix, prefix_tokens)
    t.fill(B, bs - 1)                           # one token short of a boundary
    C = t.both("seq_fork", A)                   # shares A's part-filled block
    D_ = t.both("seq_new")
    assert t.both("seq_match_prefix", D_, hashes + [0xdead]) == len(prefix)   # live hits
    E = t.both("seq_new")
    t.fill(E, bs)                               # one full private block
    eb = t.pool.seq_blocks(E)[0]
    assert t.both("cache_block", eb, 0xE0)
    t.both("seq_free", E)                       # freed, content and hash kept
    F = t.both("seq_new")
    assert t.both("seq_match_prefix", F, [0xE0]) == 1   # revived from the free queue
    assert t.pool.seq_blocks(F) == [eb]
    seqs = [A, B, C, D_, F, owner]

    cows = 0
    for step in range(steps):
        if step == 6:
            seqs.append(t.both("seq_fork", B))  # B's next write copies its last block
        if step == 9:
            t.both("seq_free", C)               # A's old block loses its last sharer
            seqs.remove(C)
        if step == 12:
            G = t.both("seq_new")
            assert t.both("seq_match_prefix", G, hashes[:2]) == 2
            t.fill(G, 1)
            seqs.append(G)
        S = len(seqs)
        ids = torch.tensor(seqs, dtype=torch.int64)
        slots = torch.empty(S, dtype=torch.int64)
        cow = torch.empty((S, 2), dtype=torch.int32)
        tables = torch.empty((S, MB), dtype=torch.int32)
        lens = torch.empty(S, dtype=torch.int32)
        pairs = t.pool.step(ids, MB, slots, cow, tables, lens).clone()
        m_slots, m_pairs = t.model.seq_append_batch(seqs)
        m_tables, m_lens = t.model.build_block_tables(seqs, MB)
        assert slots.tolist() == m_slots and pairs.tolist() == [list(p) for p in m_pairs]
        assert tables.tolist() == m_tables and lens.tolist() == m_lens
        cows += len(m_pairs)

        q = _draw((S, Hq, D), q_dtype, g)
        kn = _draw((S, Hkv, D), q_dtype, g)
        vn = _draw((S, Hkv, D), q_dtype, g)
        # GPU: copy-on-write, append, attend (two ways)
        if pairs.numel():
            pa.pa_copy_blocks(kc_d, vc_d, pairs)
        pa.pa_reshape_and_cache(kn.cuda(), vn.cuda(), kc_d, vc_d, slots.cuda(), k_scale, v_scale)
        qd, td, ld = q.cuda(), tables.cuda(), lens.cuda()
        max_ctx = int(lens.max())
        part = 0 if step % 3 == 0 else 2 * bs
        nbw = pa.pa_decode_workspace_size(S, Hq, D, max_ctx, part)
        ws = torch.empty(max(nbw, 16), dtype=torch.uint8, device="cuda")
        out = torch.full_like(qd, float("nan"))
        pa.pa_decode(out, qd, kc_d, vc_d, td, ld, max_ctx, scale, k_scale, v_scale, part,
                     ws if nbw else None)
        nbs = pa.pa_decode_shared_prefix_workspace_size(S, Hq, Hkv, D, bs, max_ctx,
                                                        prefix_tokens, kc_d.dtype)
        ws2 = torch.empty(max(nbs, 16), dtype=torch.uint8, device="cuda")
        out2 = torch.full_like(qd, float("nan"))
        pa.pa_decode_shared_prefix(out2, qd, kc_d, vc_d, td, ld, max_ctx, scale, prefix_tokens,
                                   ws2 if nbs else None, k_scale, v_scale)
        torch.cuda.synchronize()
        assert pa.pa_device_status() == 0, f"step {step}: device error"
        # oracle: the same step on the model's tables
        if m_pairs:
            k_o, v_o = oracle.copy_blocks(k_o, v_o, torch.tensor(m_pairs, dtype=torch.int32))
        k_o, v_o = oracle.reshape_and_cache(kn, vn, q_dtype, k_o, v_o, kv_dtype,
                                            torch.tensor(m_slots, dtype=torch.int64), bs,
                                            k_scale, v_scale)
        assert np.array_equal(oracle.raw(kc_d.cpu()), k_o), f"step {step}: key cache"
        assert np.array_equal(oracle.raw(vc_d.cpu()), v_o), f"step {step}: value cache"
        want = oracle.paged_decode(q, q_dtype, k_o, v_o, kv_dtype,
                                   torch.tensor(m_tables, dtype=torch.int32),
                                   torch.tensor(m_lens, dtype=torch.int32), scale,
                                   k_scale, v_scale)
        for name, got in (("pa_decode", out), ("pa_decode_shared_prefix", out2)):
            g64 = got.cpu().to(torch.float64).numpy()
            assert np.isfinite(g64).all(), f"step {step} {name}: non-finite output"
            err = np.abs(g64 - want).max()
            assert err <= TOL[kv_dtype], f"step {step} {name}: max abs error {err:.3g}"
    # the scenario did exercise what it was built for
    assert cows >= 2
    assert t.pool.stats()["cache_hits"] == t.model.cache_hits >= 6
    t.pool.close()
