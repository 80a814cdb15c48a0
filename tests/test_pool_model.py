"""Pins for the oracle's block-pool model, from the examples the pages print.

* "01. PagedAttention 详解" §3: request A's table is 42, 17, 99 for tokens
  0..47 at block size 16 (tests/golden/block_table_example.json).
* same page §6: A and B share 42 and 17 (ref_cnt 2), 99 and 88 are private
  (ref_cnt 1) (tests/golden/shared_blocks_example.json).
* same page §10 / self-check 2: 100000 tokens at block size 16 need 6250 int32
  entries, 25000 bytes (tests/golden/table_size_facts.json).
* "PagedAttention 机制" §5.3.2 / §5.3.4 and self-check 3 of the other page:
  ceil-div block counts, out-of-blocks error, free at count 0, FIFO reuse
  (tests/golden/allocator_rules.json).
"""
import numpy as np
import pytest

from oracle.pool_model import BadIndex, InvalidArg, OutOfBlocks, PoolError, PoolModel


def _pool_with_queue(nb, bs, order):
    """A pool whose free queue holds exactly ``order`` (all other blocks in use)."""
    p = PoolModel(nb, bs)
    held = [p.alloc() for _ in range(nb)]
    assert held == list(range(nb))
    for b in order:
        p.free(b)
    return p


def test_page_block_table_example(golden):
    g = golden("block_table_example.json")
    p = _pool_with_queue(100, g["block_size"], g["table"])
    a = p.seq_new()
    slots = [p.seq_append(a)[0] for _ in range(g["num_tokens"])]
    tables, lens = p.build_block_tables([a], 4)
    assert tables[0][:3] == g["table"] and tables[0][3] == -1 and lens == [48]
    for (lo, hi), blk in zip(g["token_ranges"], g["table"]):
        for i in range(lo, hi + 1):
            assert slots[i] == blk * 16 + i % 16


def test_page_shared_blocks_example(golden):
    g = golden("shared_blocks_example.json")
    bs = g["block_size"]
    p = _pool_with_queue(100, bs, [42, 17, 99, 88])
    a = p.seq_new()
    for _ in range(48):
        p.seq_append(a)
    b = p.seq_new()
    p.seq_share_prefix(b, g["table_a"][:2], 2 * bs)
    for _ in range(16):
        assert p.seq_append(b)[1:] == (-1, -1)     # a new block, no copy
    tables, _ = p.build_block_tables([a, b], 3)
    assert tables == [g["table_a"], g["table_b"]]
    for blk, r in g["ref_cnt"].items():
        assert p.ref[int(blk)] == r


def test_page_table_size_facts(golden):
    g = golden("table_size_facts.json")
    p = PoolModel(7000, g["block_size"])
    s = p.seq_new()
    for _ in range(g["num_tokens"]):
        p.seq_append(s)
    tables, _ = p.build_block_tables([s], g["entries"])
    t = np.asarray(tables, dtype=np.int32)
    assert t.shape == (1, g["entries"]) and t.nbytes == g["table_bytes"]
    assert (t >= 0).all()
    # the per-token KV bytes the measurement formula uses, at the page's sizes
    from workloads import DecodeConfig, kv_bytes_per_token
    cfg = DecodeConfig("page", 1, 32, 32, 128, 16, "f16", "f16", 1, 1)  # hidden 4096
    assert kv_bytes_per_token(cfg) == g["kv_bytes_per_token_per_layer_hidden4096_fp16"]
    assert kv_bytes_per_token(cfg) * g["layers"] == g["kv_bytes_per_token_all_layers"]


def test_blocks_needed_is_ceil_div(golden):
    g = golden("allocator_rules.json")
    for n, bs, want in g["blocks_needed"]:
        p = PoolModel(want + 1, bs)
        s = p.seq_new()
        for _ in range(n):
            p.seq_append(s)
        assert len(p.seq_blocks(s)) == want


def test_allocator_rules():
    p = PoolModel(3, 16)
    assert [p.alloc() for _ in range(3)] == [0, 1, 2]
    with pytest.raises(OutOfBlocks):
        p.alloc()
    p.incr_ref(1)
    p.free(1)
    assert p.ref[1] == 1 and 1 not in p.free_queue
    p.free(2)
    p.free(1)
    p.free(0)
    assert list(p.free_queue) == [2, 1, 0]        # tail order = order counts hit 0
    assert p.alloc() == 2                         # head first
    with pytest.raises(PoolError):
        p.free(1)                                 # already free
    with pytest.raises(PoolError):
        p.incr_ref(0)                             # a free block cannot be shared
    with pytest.raises(BadIndex):
        p.free(3)


def test_out_of_blocks_leaves_state_unchanged():
    p = PoolModel(2, 4)
    s = p.seq_new()
    for _ in range(8):
        p.seq_append(s)
    before = (list(p.free_queue), list(p.ref), p.seq_len(s))
    with pytest.raises(OutOfBlocks):
        p.seq_append(s)
    assert (list(p.free_queue), list(p.ref), p.seq_len(s)) == before


def test_copy_on_write_on_shared_last_block():
    p = PoolModel(8, 4)
    a = p.seq_new()
    for _ in range(6):                 # blocks 0 (full), 1 (2 of 4)
        p.seq_append(a)
    b = p.seq_fork(a)                  # parallel sampling: child shares both
    assert p.ref[0] == 2 and p.ref[1] == 2
    slot, src, dst = p.seq_append(b)   # b writes into shared block 1 -> copy
    assert (src, dst) == (1, 2) and slot == 2 * 4 + 2
    assert p.ref[1] == 1 and p.ref[2] == 1 and p.seq_blocks(b) == [0, 2]
    slot, src, dst = p.seq_append(a)   # a is now the only holder of 1: no copy
    assert (src, dst) == (-1, -1) and slot == 1 * 4 + 2
    assert p.stats()["cow_copies"] == 1
    p.seq_free(a)
    assert p.ref[0] == 1 and p.ref[1] == 0 and list(p.free_queue)[-1] == 1
    p.seq_free(b)
    assert sum(p.ref) == 0 and sorted(p.free_queue) == list(range(8))


# -- prefix cache: "01. PagedAttention 详解" self-check 3 and summary (hash hit
#    -> ref_cnt++, LRU reuse of freed blocks); prefix_hashing as named in the
#    intelliparadigm PagedAttention article §5.1 ---------------------------------

def _filled_seq(p, ntok):
    s = p.seq_new()
    for _ in range(ntok):
        p.seq_append(s)
    return s


def test_cache_hit_on_a_live_block_adds_a_reference():
    p = PoolModel(8, 4)
    a = _filled_seq(p, 8)                        # blocks 0, 1 full
    assert p.cache_block(0, 111) and p.cache_block(1, 222)
    assert p.cache_lookup(111) == 0              # _get_cached_block: ref_cnt++
    assert p.ref[0] == 2 and p.ref[1] == 1
    assert p.cache_lookup(999) == -1 and p.ref == [2, 1] + [0] * 6
    assert p.stats()["cache_hits"] == 1 and p.stats()["shared"] == 1
    p.free(0)
    p.seq_free(a)
    assert p.ref[0] == 0 and list(p.free_queue)[-2:] == [0, 1]


def test_freed_cached_block_is_revived_from_the_queue():
    p = PoolModel(4, 4)
    a = _filled_seq(p, 8)                        # blocks 0, 1
    p.cache_block(0, 7)
    p.seq_free(a)                                # both counts reach 0, content kept
    assert list(p.free_queue) == [2, 3, 0, 1]
    assert p.cache_lookup(7) == 0                # leaves the middle of the queue
    assert p.ref[0] == 1 and list(p.free_queue) == [2, 3, 1]
    assert p.cached == {7: 0}


def test_reuse_from_the_queue_head_evicts_the_least_recently_freed():
    p = PoolModel(3, 2)
    x, y = _filled_seq(p, 2), _filled_seq(p, 2)  # blocks 0 and 1
    p.cache_block(0, 10)
    p.cache_block(1, 11)
    p.seq_free(x)                                # 0 freed first ...
    p.seq_free(y)                                # ... then 1
    assert list(p.free_queue) == [2, 0, 1]
    assert p.alloc() == 2                        # never cached: no eviction
    assert p.alloc() == 0                        # reuse evicts hash 10
    assert p.cache_lookup(10) == -1
    assert p.cache_lookup(11) == 1               # the more recently freed survives
    assert p.stats()["cached"] == 1


def test_a_hash_names_one_block_and_writes_drop_it():
    p = PoolModel(6, 4)
    a = _filled_seq(p, 4)
    b = _filled_seq(p, 4)
    assert p.cache_block(0, 5)
    assert not p.cache_block(1, 5)               # same content elsewhere: first stays
    assert p.cache_block(0, 5)                   # idempotent
    with pytest.raises(InvalidArg):
        p.cache_block(0, 6)
    with pytest.raises(PoolError):
        p.cache_block(4, 6)                      # a free block cannot be registered
    # a partial block registered by the caller loses its hash once written alone
    c = _filled_seq(p, 2)
    blk = p.seq_blocks(c)[0]
    p.cache_block(blk, 77)
    p.seq_append(c)
    assert p.cache_lookup(77) == -1
    # ... but a shared one is copied first and keeps it
    p.cache_block(blk, 78)
    d = p.seq_fork(c)
    slot, src, dst = p.seq_append(d)
    assert src == blk and p.cache_lookup(78) == blk
    del a, b


def test_match_prefix_takes_the_leading_hits_only():
    bs = 4
    p = PoolModel(10, bs)
    a = _filled_seq(p, 3 * bs + 1)               # blocks 0, 1, 2 full, 3 partial
    for i, h in enumerate((100, 101, 102)):
        p.cache_block(i, h)
    p.seq_free(a)
    b = p.seq_new()
    assert p.seq_match_prefix(b, [100, 101, 555, 102]) == 2
    assert p.seq_blocks(b) == [0, 1] and p.seq_len(b) == 2 * bs
    assert p.ref[:4] == [1, 1, 0, 0]
    slot, src, dst = p.seq_append(b)             # next token opens a fresh block
    assert (src, dst) == (-1, -1) and slot // bs not in (0, 1, 2)
    with pytest.raises(InvalidArg):
        p.seq_match_prefix(b, [102])             # only into an empty sequence
    c = p.seq_new()
    assert p.seq_match_prefix(c, [100, 101, 102]) == 3
    assert p.ref[:3] == [2, 2, 1]
