"""Host-side checks of the C ABI (no GPU needed).

* The shared library loads and exports every function include/pa.h declares.
* Argument checks reject bad calls before anything reaches a device.
* The C++ block pool replays the pages' examples and long random call
  sequences exactly like the oracle's pool model (same slots, copy-on-write
  pairs, tables, reference counts, free order and errors).
"""
import os
import random
import re

import pytest
import torch

import paged_kv_cache_338_b200 as pa
from oracle.pool_model import PoolError, PoolModel

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 20
    L = pa.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing
    assert pa.pa_version() == 10000


def test_binding_constants_match_the_header():
    """The few #defines the binding mirrors have the header's values."""
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    assert re.search(r"#define PA_PARTITION_BALANCED \(-1\)", src)
    assert pa.PA_PARTITION_BALANCED == -1
    m = re.search(r"#define PA_DECODE_NOALLOC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", src)
    assert m and pa.PA_DECODE_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_no_symbol_leaks_beyond_the_abi():
    # the static CUDA runtime stays private to the library
    out = os.popen(f"nm -D --defined-only {pa.LIB_PATH}").read().split("\n")
    exported = {l.split()[-1] for l in out if l.strip() and l.split()[1] in "TtWw"}
    extra = {n for n in exported if not n.startswith("pa_")}
    assert not {n for n in extra if n.startswith("cuda")}, sorted(extra)[:10]


def _bad(fn, *a, status="PA_ERR_INVALID_ARG"):
    with pytest.raises(pa.PaError) as e:
        fn(*a)
    assert e.value.status == status, str(e.value)


def test_host_argument_checks():
    L = pa.lib()
    nb = torch.zeros(1, dtype=torch.int64)
    # decode: bad dtype, group not a divisor, block size, partition not a multiple of bs
    assert L.pa_decode(None, None, 7, None, None, 2, None, 1, None, 1, 8, 2, 128, 16, 10, 16,
                       1.0, 1.0, 1.0, 0, None, 0, None) == 1
    assert L.pa_decode(None, None, 2, None, None, 2, None, 1, None, 1, 6, 4, 128, 16, 10, 16,
                       1.0, 1.0, 1.0, 0, None, 0, None) == 1
    assert L.pa_decode(None, None, 2, None, None, 2, None, 1, None, 1, 8, 2, 128, 12, 10, 16,
                       1.0, 1.0, 1.0, 0, None, 0, None) == 2
    assert L.pa_decode(None, None, 2, None, None, 2, None, 1, None, 1, 8, 2, 128, 16, 10, 16,
                       1.0, 1.0, 1.0, 24, None, 0, None) == 1
    # non-fp8 caches take unit scales only; fp8 needs f16/bf16 q
    assert L.pa_decode(None, None, 2, None, None, 2, None, 1, None, 1, 8, 2, 128, 16, 10, 16,
                       1.0, 2.0, 1.0, 0, None, 0, None) == 1
    assert L.pa_decode(None, None, 0, None, None, 3, None, 1, None, 1, 8, 2, 128, 16, 10, 16,
                       1.0, 1.0, 1.0, 0, None, 0, None) == 2
    # S == 0 is a no-op even without pointers
    assert L.pa_decode(None, None, 2, None, None, 2, None, 1, None, 0, 8, 2, 128, 16, 10, 16,
                       1.0, 1.0, 1.0, 0, None, 0, None) == 0
    # split-K without enough workspace
    assert L.pa_decode(16, 16, 2, 16, 16, 2, 16, 8, 16, 1, 8, 2, 128, 16, 10, 1000,
                       1.0, 1.0, 1.0, 256, None, 0, None) == 1
    assert "workspace" in pa.pa_last_error()
    # append: unsupported dtype pair, scales, zero tokens is a no-op
    assert L.pa_reshape_and_cache(None, None, 2, None, None, 1, None, 4, 8, 128, 16, 10,
                                  1.0, 1.0, None) == 2
    assert L.pa_reshape_and_cache(None, None, 2, None, None, 3, None, 4, 8, 128, 16, 10,
                                  0.0, 1.0, None) == 1
    assert L.pa_reshape_and_cache(None, None, 2, None, None, 2, None, 0, 8, 128, 16, 10,
                                  1.0, 1.0, None) == 0


def test_decode_select_modes():
    """Every documented bit combination is accepted (0..127, bits 8, 16, 32 and
    64 included) and anything else refused; the default is restored afterwards."""
    try:
        for mode in range(128):
            pa.pa_decode_select(mode)
        for bad in (-1, 128, 256):
            _bad(pa.pa_decode_select, bad)
    finally:
        pa.pa_decode_select(pa.DECODE_DEFAULT)


def test_partition_group_plan():
    """The grouped split-K plan (host logic, 148 SMs): the 4 x 100k bf16
    workload with 512-token partitions streams 4 partitions per CTA of four kv
    heads (392 CTAs, one wave of 3 per SM), and 16 with one kv head per CTA
    (416 CTAs); multi-head attention (the tensor-core consumer too) groups as
    well; long partitions, a single pass, the CUDA-core consumer and fp32
    caches stay at one; the test bit forces three.  Shapes pa_decode refuses
    are refused here with the same codes."""
    bf, f8, f16, f32 = torch.bfloat16, torch.float8_e4m3fn, torch.float16, torch.float32

    def grp(S, Hq, Hkv, D, ct, ctx, part, sms, bs=16, qt=None):
        qt = qt if qt is not None else (bf if ct == f8 else ct)
        return pa.pa_decode_partition_group(S, Hq, Hkv, D, bs, qt, ct, ctx, part, sms)
    try:
        pa.pa_decode_select(pa.DECODE_DEFAULT)
        assert grp(4, 32, 8, 128, bf, 100000, 512, 148) == 4
        assert grp(4, 32, 8, 128, f8, 100000, 512, 148) == 4
        assert grp(128, 32, 8, 128, bf, 8192, 2048, 148) == 1   # 1 MB partitions
        assert grp(4, 32, 8, 128, bf, 100000, 0, 148) == 1      # single pass
        assert grp(4, 32, 32, 128, f16, 100000, 512, 148) > 1   # MHA: tensor-core consumer
        assert grp(4, 32, 8, 128, f32, 100000, 512, 148) == 1
        assert grp(4, 32, 8, 128, bf, 400, 512, 148) == 1       # one partition
        # never more partitions per CTA than a sequence has; no part-filled
        # second wave when the groups would fit one
        for S, ctx in ((1, 20000), (2, 50000), (16, 30000), (64, 9000)):
            g = grp(S, 32, 8, 128, bf, ctx, 256, 148)
            parts = -(-ctx // 256)
            ctas = S * 2 * (-(-parts // g))                      # two CTAs of four kv heads
            assert 1 <= g <= parts
            assert not (444 < ctas < 2 * 444 and S * 2 * (-(-parts // (g + 1))) <= 444)
        pa.pa_decode_select(pa.DECODE_DEFAULT | pa.DECODE_ONE_HEAD_PER_CTA)
        assert grp(4, 32, 8, 128, bf, 100000, 512, 148) == 16
        pa.pa_decode_select(pa.DECODE_DEFAULT | pa.DECODE_GROUP_PARTITIONS)
        assert grp(4, 32, 8, 128, bf, 100000, 512, 148) == 3
        pa.pa_decode_select(pa.DECODE_DEFAULT | pa.DECODE_SIMT_ONLY)
        assert grp(4, 32, 8, 128, bf, 100000, 512, 148) == 1
    finally:
        pa.pa_decode_select(pa.DECODE_DEFAULT)
    G = pa.pa_decode_partition_group
    # 32 % 6
    _bad(G, 4, 32, 6, 128, 16, bf, bf, 1000, 512, 148)
    # head dim
    _bad(G, 4, 32, 8, 96, 16, bf, bf, 1000, 512, 148, status="PA_ERR_UNSUPPORTED")
    # group of 3
    _bad(G, 4, 24, 8, 128, 16, bf, bf, 1000, 512, 148, status="PA_ERR_UNSUPPORTED")
    # partition % bs
    _bad(G, 4, 32, 8, 128, 16, bf, bf, 1000, 500, 148)
    # block size
    _bad(G, 4, 32, 8, 128, 12, bf, bf, 1000, 480, 148, status="PA_ERR_UNSUPPORTED")
    # q f16, cache bf16
    _bad(G, 4, 32, 8, 128, 16, f16, bf, 1000, 512, 148, status="PA_ERR_UNSUPPORTED")
    # fp8 queries
    _bad(G, 4, 32, 8, 128, 16, f8, f8, 1000, 512, 148, status="PA_ERR_UNSUPPORTED")
    # fp32 q, fp8 cache
    _bad(G, 4, 32, 8, 128, 16, f32, f8, 1000, 512, 148, status="PA_ERR_UNSUPPORTED")
    # balanced: no plan
    _bad(G, 4, 32, 8, 128, 16, bf, bf, 1000, -1, 148)


def test_copy_blocks_host_rejections():
    kc = torch.zeros((8, 16, 2, 64), dtype=torch.bfloat16)   # host memory: never launched
    for bad in ([[1, 2], [3, 2]], [[1, 2], [2, 4]], [[1, 8]], [[-1, 3]]):
        _bad(pa.pa_copy_blocks, kc, kc, bad)
    pa.pa_copy_blocks(kc, kc, [])   # no pairs: nothing to do


def test_workspace_size_and_suggested_partition():
    assert pa.pa_decode_workspace_size(4, 32, 128, 100000, 512) == 4 * 32 * 196 * (8 + 4 * 128)
    assert pa.pa_decode_workspace_size(4, 32, 128, 512, 512) == 0
    assert pa.pa_decode_workspace_size(4, 32, 128, 100000, 0) == 0
    p = pa.pa_decode_suggest_partition(8, 16, [100000] * 4)
    assert p > 0 and p % 16 == 0 and p < 100000
    assert pa.pa_decode_suggest_partition(32, 16, [64] * 4096) == 0


# ------------------------------------------------------------------ pool

def _run_both(model, pool, op, *args):
    err_m = err_p = None
    try:
        rm = getattr(model, op)(*args)
    except PoolError as e:
        err_m, rm = e.status, None
    try:
        rp = getattr(pool, op)(*args)
    except pa.PaError as e:
        err_p, rp = e.status, None
    assert err_m == err_p, (op, args, err_m, err_p)
    return rm, rp


def test_pool_replays_page_examples(golden):
    g = golden("shared_blocks_example.json")
    pool = pa.BlockPool(100, 16)
    held = [pool.alloc() for _ in range(100)]
    assert held == list(range(100))
    for b in (42, 17, 99, 88):
        pool.free(b)
    a = pool.seq_new()
    for _ in range(48):
        pool.seq_append(a)
    b = pool.seq_new()
    pool.seq_share_prefix(b, [42, 17], 32)
    for _ in range(16):
        assert pool.seq_append(b)[1:] == (-1, -1)
    t, lens = pool.build_block_tables([a, b], 3)
    assert t.tolist() == [g["table_a"], g["table_b"]] and lens.tolist() == [48, 48]
    for blk, r in g["ref_cnt"].items():
        assert pool.ref(int(blk)) == r
    # 100000 tokens -> 6250 int32 entries (25000 bytes)
    f = golden("table_size_facts.json")
    big = pa.BlockPool(7000, 16)
    s = big.seq_new()
    for _ in range(f["num_tokens"]):
        big.seq_append(s)
    t, lens = big.build_block_tables([s], f["entries"])
    assert t.numel() * 4 == f["table_bytes"] and int(lens[0]) == f["num_tokens"]
    assert (t >= 0).all()


@pytest.mark.parametrize("seed", range(6))
def test_pool_matches_model_on_random_call_sequences(seed):
    rnd = random.Random(seed)
    nb, bs = rnd.choice([(12, 4), (40, 8), (64, 16), (7, 32)])
    model, pool = PoolModel(nb, bs), pa.BlockPool(nb, bs)
    live = []
    for step in range(1500):
        r = rnd.random()
        if r < 0.08 or not live:
            m, p = _run_both(model, pool, "seq_new")
            assert m == p
            live.append(m)
        elif r < 0.55:
            s = rnd.choice(live)
            m, p = _run_both(model, pool, "seq_append", s)
            assert m == p
        elif r < 0.62:
            m, p = _run_both(model, pool, "seq_fork", rnd.choice(live))
            assert m == p
            if m is not None:
                live.append(m)
        elif r < 0.70 and len(live) > 1:
            s = live.pop(rnd.randrange(len(live)))
            _run_both(model, pool, "seq_free", s)
        elif r < 0.75:
            s = rnd.choice(live)
            if model.seq_len(s) > 0:
                src = model.seq_blocks(s)
                n = rnd.randint(1, len(src))
                t = model.seq_new()
                assert pool.seq_new() == t
                live.append(t)
                ntok = min(model.seq_len(s), n * bs)
                _run_both(model, pool, "seq_share_prefix", t, src[:n], ntok)
        elif r < 0.80:
            _run_both(model, pool, "free", rnd.randrange(-1, nb + 1))
        elif r < 0.85:
            _run_both(model, pool, "incr_ref", rnd.randrange(nb))
        elif r < 0.88:
            m, p = _run_both(model, pool, "alloc")
            assert m == p
        else:
            _run_both(model, pool, "seq_append", 10_000 + step)     # unknown sequence
        assert [pool.ref(b) for b in range(nb)] == model.ref
        st = pool.stats()
        ms = model.stats()
        for k in ("free", "used", "shared"):
            assert st[k if k != "free" else "free_blocks"] == ms[k] if k == "free" else \
                st[k + "_blocks"] == ms[k]
        assert st["cow_copies"] == ms["cow_copies"] and st["num_seqs"] == ms["num_seqs"]
    mb = max([len(model.seq_blocks(s)) for s in live] + [1])
    tm, lm = model.build_block_tables(live, mb)
    tp, lp = pool.build_block_tables(live, mb)
    assert tp.tolist() == tm and lp.tolist() == lm
    # drain: free order must match (observed through the next allocations)
    for s in live:
        _run_both(model, pool, "seq_free", s)
    while model.free_queue:
        m, p = _run_both(model, pool, "alloc")
        assert m == p
    _run_both(model, pool, "alloc")


@pytest.mark.parametrize("seed", range(3))
def test_pool_batch_append_matches_model(seed):
    rnd = random.Random(100 + seed)
    nb, bs = 64, 8
    model, pool = PoolModel(nb, bs), pa.BlockPool(nb, bs)
    seqs = []
    for _ in range(6):
        s = model.seq_new()
        assert pool.seq_new() == s
        seqs.append(s)
    for step in range(80):
        if rnd.random() < 0.15:            # a sampling fork shares the last block
            parent = rnd.choice(seqs)
            c = model.seq_fork(parent)
            assert pool.seq_fork(parent) == c
            seqs.append(c)
        batch = rnd.sample(seqs, rnd.randint(1, len(seqs)))
        try:
            ms, mp = model.seq_append_batch(batch)
            merr = None
        except PoolError as e:
            merr = e.status
        try:
            ps, pp = pool.seq_append_batch(batch)
            perr = None
        except pa.PaError as e:
            perr = e.status
        assert merr == perr
        if merr is None:
            assert ps.tolist() == ms and pp.tolist() == [list(x) for x in mp]
        assert [pool.ref(b) for b in range(nb)] == model.ref
    with pytest.raises(pa.PaError):
        pool.seq_append_batch([seqs[0], seqs[0]])      # repeated sequence


@pytest.mark.parametrize("seed", range(6))
def test_prefix_cache_matches_model_on_random_call_sequences(seed):
    """Hash registration, hits on live and freed blocks, LRU eviction through
    allocation, and prefix matching, replayed against the oracle's model."""
    rnd = random.Random(1000 + seed)
    nb, bs = rnd.choice([(16, 4), (48, 8), (9, 16)])
    model, pool = PoolModel(nb, bs), pa.BlockPool(nb, bs)
    hashes = [rnd.getrandbits(64) for _ in range(24)]
    live = []
    for step in range(1500):
        r = rnd.random()
        if r < 0.08 or not live:
            m, p = _run_both(model, pool, "seq_new")
            assert m == p
            live.append(m)
        elif r < 0.45:
            m, p = _run_both(model, pool, "seq_append", rnd.choice(live))
            assert m == p
        elif r < 0.50:
            m, p = _run_both(model, pool, "seq_fork", rnd.choice(live))
            assert m == p
            if m is not None:
                live.append(m)
        elif r < 0.60 and len(live) > 1:
            _run_both(model, pool, "seq_free", live.pop(rnd.randrange(len(live))))
        elif r < 0.72:
            s = rnd.choice(live)
            blocks = model.seq_blocks(s)
            full = model.seq_len(s) // bs
            if full:
                i = rnd.randrange(full)
                m, p = _run_both(model, pool, "cache_block", blocks[i], rnd.choice(hashes))
                assert m == p
        elif r < 0.80:
            m, p = _run_both(model, pool, "cache_lookup", rnd.choice(hashes))
            assert m == p
            if m is not None and m >= 0:
                _run_both(model, pool, "free", m)
        elif r < 0.88:
            t, tp = _run_both(model, pool, "seq_new")
            assert t == tp
            live.append(t)
            hs = [rnd.choice(hashes) for _ in range(rnd.randint(0, 4))]
            m, p = _run_both(model, pool, "seq_match_prefix", t, hs)
            assert m == p
        elif r < 0.92:
            m, p = _run_both(model, pool, "alloc")
            assert m == p
            if m is not None:
                _run_both(model, pool, "free", m)
        else:
            _run_both(model, pool, "cache_block", rnd.randrange(-1, nb + 1), hashes[0])
        assert [pool.ref(b) for b in range(nb)] == model.ref
        st, ms = pool.stats(), model.stats()
        assert (st["free_blocks"], st["cached_blocks"], st["cache_hits"]) == \
            (ms["free"], ms["cached"], ms["cache_hits"])
    for s in live:
        assert pool.seq_blocks(s) == model.seq_blocks(s)
        _run_both(model, pool, "seq_free", s)
    while len(model.free_queue):      # same LRU order, same surviving hashes
        for h in hashes:
            m, p = _run_both(model, pool, "cache_lookup", h)
            assert m == p
            if m >= 0:
                _run_both(model, pool, "free", m)
        m, p = _run_both(model, pool, "alloc")
        assert m == p


def test_prefix_cache_argument_checks():
    pool = pa.BlockPool(4, 4)
    s = pool.seq_new()
    for _ in range(4):
        pool.seq_append(s)
    _bad(pool.cache_block, 9, 1, status="PA_ERR_BAD_INDEX")
    _bad(pool.cache_block, 3, 1, status="PA_ERR_REFCOUNT")
    assert pool.cache_block(0, 1) and pool.cache_block(0, 1)
    _bad(pool.cache_block, 0, 2)
    _bad(pool.seq_match_prefix, s, [1])
    _bad(pool.seq_match_prefix, 99, [1], status="PA_ERR_BAD_INDEX")
    _bad(pool.seq_blocks, 99, status="PA_ERR_BAD_INDEX")
    assert pool.cache_lookup(1) == 0 and pool.ref(0) == 2
    assert pool.cache_lookup(2 ** 64 - 1) == -1
    assert pool.stats()["cache_hits"] == 1


def test_prefill_host_argument_checks():
    L = pa.lib()
    # (out, q, q_dt, kc, vc, cache_dt, bt, MB, lens, qs, S, T, Hq, Hkv, D, bs, NB, maxq, scale, st)
    base = [16, 16, 2, 16, 16, 2, 16, 4, 16, 16, 2, 10, 8, 2, 128, 16, 10, 8, 0.1, None]

    def call(**kw):
        a = list(base)
        names = ["out", "q", "q_dt", "kc", "vc", "cache_dt", "bt", "MB", "lens", "qs", "S", "T",
                 "Hq", "Hkv", "D", "bs", "NB", "maxq", "scale", "st"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return L.pa_prefill(*a)

    assert call(q_dt=2, cache_dt=3) == 2          # fp8 cache: the tensor cores take one type
    assert call(q_dt=0, cache_dt=0) == 2          # fp32
    assert call(q_dt=1, cache_dt=2) == 2          # mixed
    assert call(q_dt=9) == 1                      # unknown dtype
    assert call(D=256) == 2 and call(D=96) == 2
    assert call(bs=64) == 2
    assert call(Hq=6, Hkv=2) == 2                 # group 3
    assert call(Hq=7, Hkv=2) == 1                 # not a divisor
    assert call(scale=float("inf")) == 1 and call(scale=0.0) == 1 and call(scale=-0.1) == 1
    assert call(out=None) == 1
    assert call(q=24) == 1                        # misaligned
    assert call(S=70000) == 2                     # grid limit
    # nothing to do: no sequences, no tokens or empty chunks
    assert call(S=0, out=None, q=None) == 0
    assert call(T=0, out=None, q=None) == 0
    assert call(maxq=0, out=None) == 0


def test_shared_prefix_host_argument_checks():
    L = pa.lib()
    # (out, q, q_dt, kc, vc, cache_dt, bt, MB, lens, S, Hq, Hkv, D, bs, NB, max_ctx, scale,
    #  k_scale, v_scale, prefix, ws, ws_bytes, stream)
    base = [16, 16, 2, 16, 16, 2, 16, 64, 16, 4, 32, 8, 128, 16, 100, 2000, 0.1, 1.0, 1.0, 512,
            16, 1 << 30, None]
    names = ["out", "q", "q_dt", "kc", "vc", "cache_dt", "bt", "MB", "lens", "S", "Hq", "Hkv",
             "D", "bs", "NB", "max_ctx", "scale", "ks", "vs", "prefix", "ws", "wsb", "st"]

    def call(**kw):
        a = list(base)
        for k, v in kw.items():
            a[names.index(k)] = v
        return L.pa_decode_shared_prefix(*a)

    assert call(q_dt=0, cache_dt=0) == 2            # fp32
    assert call(cache_dt=3, D=64) == 2              # fp8 rows of 64 bytes
    assert call(D=256) == 2
    assert call(prefix=100) == 1                    # not a multiple of bs
    assert call(prefix=64 * 16 + 16) == 1           # beyond MB * bs
    assert call(Hq=24, Hkv=8) == 2                  # group 3
    assert call(scale=0.0) == 1
    assert call(S=0, out=None) == 0
    assert call(ws=None) == 1 and "workspace" in pa.pa_last_error()
    rec = lambda parts: -(-(4 * 32 * parts * (8 + 4 * 128)) // 256) * 256
    # suffixes of at most 4096 tokens: the 2 prefix records only (256-token chunks)
    n = pa.pa_decode_shared_prefix_workspace_size(4, 32, 8, 128, 16, 2000, 512, torch.bfloat16)
    assert n == rec(2)
    n8 = pa.pa_decode_shared_prefix_workspace_size(4, 32, 8, 128, 16, 2000, 512,
                                                   torch.float8_e4m3fn)
    assert n8 == n + 2 * 512 * 8 * 128 * 2                          # + 16-bit K, V prefix copies
    # longer suffixes: every 256-token partition of max_ctx has a record
    assert pa.pa_decode_shared_prefix_workspace_size(4, 32, 8, 128, 16, 10000, 512,
                                                     torch.bfloat16) == rec(40)
    assert pa.pa_decode_shared_prefix_workspace_size(4, 32, 8, 128, 16, 300, 512,
                                                     torch.bfloat16) == 0   # plain decode


@pytest.mark.parametrize("seed", range(3))
def test_pool_step_equals_append_then_pack(seed):
    """pa_pool_step = seq_append_batch + build_block_tables, all or nothing."""
    rnd = random.Random(500 + seed)
    nb, bs, MB = 80, 8, (3, 12, 5)[seed]          # small MB: the table-width rule fires
    a, b = pa.BlockPool(nb, bs), pa.BlockPool(nb, bs)
    seqs = []
    for _ in range(6):
        s1, s2 = a.seq_new(), b.seq_new()
        assert s1 == s2
        seqs.append(s1)
    for step in range(60):
        if rnd.random() < 0.1:
            parent = rnd.choice(seqs)
            c1, c2 = a.seq_fork(parent), b.seq_fork(parent)
            assert c1 == c2
            seqs.append(c1)
        batch = torch.tensor(rnd.sample(seqs, rnd.randint(1, len(seqs))), dtype=torch.int64)
        n = batch.numel()
        slots_a, cow_a = torch.empty(n, dtype=torch.int64), torch.empty((n, 2), dtype=torch.int32)
        tab_a, len_a = torch.empty((n, MB), dtype=torch.int32), torch.empty(n, dtype=torch.int32)
        try:
            pairs_a = a.step(batch, MB, slots_a, cow_a, tab_a, len_a)
            err_a = None
        except pa.PaError as e:
            err_a = e.status
        # the same through the two separate calls, guarded by the same MB rule
        fits = all(len(b.seq_blocks(int(s))) + (b.seq_len(int(s)) % bs == 0) <= MB for s in batch)
        err_b = None
        if not fits:
            err_b = "PA_ERR_INVALID_ARG"
        else:
            try:
                slots_b, pairs_b = b.seq_append_batch(batch)
                tab_b, len_b = b.build_block_tables(batch, MB)
            except pa.PaError as e:
                err_b = e.status
        assert err_a == err_b
        if err_a is None:
            assert torch.equal(slots_a, slots_b) and torch.equal(pairs_a, pairs_b)
            assert torch.equal(tab_a, tab_b) and torch.equal(len_a, len_b)
        assert [a.ref(i) for i in range(nb)] == [b.ref(i) for i in range(nb)]


def _lpt(lens, ndev):
    """Longest first (stable), each to the least loaded device (lowest on ties)."""
    order = sorted(range(len(lens)), key=lambda s: -lens[s])
    load, dev = [0] * ndev, [0] * len(lens)
    for s in order:
        d = min(range(ndev), key=lambda i: (load[i], i))
        dev[s] = d
        load[d] += lens[s]
    return dev, load


@pytest.mark.parametrize("seed", range(4))
def test_plan_shards_is_lpt_and_balanced(seed):
    """pa_plan_shards: the longest-first greedy plan exactly; every sequence on
    one device; per-device tokens add up; within Graham's 4/3 bound of the
    best split (brute force on small batches)."""
    import itertools
    g = torch.Generator().manual_seed(seed)
    for trial in range(30):
        S = int(torch.randint(0, 9, (1,), generator=g))
        nd = int(torch.randint(1, 4, (1,), generator=g))
        lens = torch.randint(0, 50, (S,), generator=g).tolist()
        dev, tok = pa.pa_plan_shards(lens, nd)
        want_dev, want_load = _lpt(lens, nd)
        assert dev.tolist() == want_dev and tok.tolist() == want_load
        if S:
            best = min(max(sum(l for l, a in zip(lens, asg) if a == d) for d in range(nd))
                       for asg in itertools.product(range(nd), repeat=S))
            assert max(want_load) <= (4 / 3 - 1 / (3 * nd)) * best + 1e-9
    big = torch.randint(1, 8193, (1024,), generator=g)
    dev, tok = pa.pa_plan_shards(big, 8)
    assert int(tok.sum()) == int(big.sum()) and int(tok.max() - tok.min()) <= 8192
    _bad(pa.pa_plan_shards, [3, 4], 0)
    _bad(pa.pa_plan_shards, [3, -1], 2)
