"""Reference model of the refcounted physical block pool -- TEST INFRASTRUCTURE ONLY.

Plain Python, one step per rule on the pages:

* "PagedAttention 机制" §5.3.4, BlockAllocator: a free list and a per-block
  reference count; allocate fails when the free list is empty, else takes a
  block and sets its count to 1; free decrements and returns the block to the
  free list when the count reaches 0; incr_ref adds a reference (sharing).
* "01. PagedAttention 详解" self-check 3 (get_new_blocks / free_blocks): the
  free list is a queue -- allocation takes from the head, a block whose count
  drops to 0 goes to the tail (least recently freed is reused first).  Where
  this and the first page's list pop() differ, the queue is taken.
* "PagedAttention 机制" §5.3.2, BlockTable.allocate: a sequence of n tokens
  holds ceil(n / block_size) blocks; a table maps logical block i to a
  physical id.
* intelliparadigm PagedAttention article §3.3, maybe_copy_block: writing into a
  block whose count is above 1 first allocates a new block, copies, drops one
  reference from the old block and continues in the new one.
* "01. PagedAttention 详解" §6 and summary: sequences may share blocks (a common
  prefix, or a fork for beam search / parallel sampling) by adding references.
* Prefix cache, "01. PagedAttention 详解" self-check 3 (a hash hit on a
  block: _get_cached_block raises its ref_cnt) and summary; the
  intelliparadigm PagedAttention article §5.1 names the same switch
  (prefix_hashing) in its OOM table: a
  full block may be registered under a hash of its content; a hit takes a
  reference on the cached block (_get_cached_block: ref_cnt++), which also
  revives a block whose count had dropped to 0 but which still sits, content
  intact, in the free queue; allocation from the head of the queue evicts the
  oldest freed block's content (LRU reuse).  Which hash names which content is
  the caller's choice.  Readings where the pages are silent: a hash names at
  most one block (registering a second block under a held hash leaves the
  first one in place); writing into a block the writer holds alone drops its
  hash, since the content changes.

Misuse raises a PoolError subclass whose ``status`` names the library's
status code: freeing a free block or sharing a free block (PA_ERR_REFCOUNT),
an unknown sequence or an out-of-range block id (PA_ERR_BAD_INDEX), malformed
requests (PA_ERR_INVALID_ARG); running out of free blocks raises OutOfBlocks
(PA_ERR_OUT_OF_BLOCKS) and leaves the state unchanged.
"""
from __future__ import annotations

from collections import Counter, OrderedDict


class PoolError(Exception):
    status = "PA_ERR_REFCOUNT"


class OutOfBlocks(PoolError):
    status = "PA_ERR_OUT_OF_BLOCKS"


class InvalidArg(PoolError):
    status = "PA_ERR_INVALID_ARG"


class BadIndex(PoolError):
    status = "PA_ERR_BAD_INDEX"


class _FreeQueue:
    """FIFO of free block ids that a prefix-cache hit can also take from the
    middle (an insertion-ordered dict used as a set)."""

    def __init__(self, items):
        self._d = OrderedDict((b, None) for b in items)

    def __len__(self):
        return len(self._d)

    def __iter__(self):
        return iter(self._d)

    def __contains__(self, b):
        return b in self._d

    def popleft(self):
        b, _ = self._d.popitem(last=False)
        return b

    def append(self, b):
        self._d[b] = None

    def remove(self, b):
        del self._d[b]


class PoolModel:
    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidArg("bad sizes")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_queue = _FreeQueue(range(num_blocks))
        self.ref = [0] * num_blocks
        self.seqs = {}            # id -> [blocks list, num tokens]
        self.next_seq = 0
        self.cow_count = 0
        self.cached = {}          # content hash -> block holding it
        self.block_hash = {}      # block -> its registered hash
        self.cache_hits = 0

    # -- blocks -----------------------------------------------------------
    def _check_block(self, b):
        if not (0 <= b < self.num_blocks):
            raise BadIndex(f"block {b} out of range")

    def alloc(self) -> int:
        if not self.free_queue:
            raise OutOfBlocks("no free blocks")
        b = self.free_queue.popleft()
        self._forget(b)           # reuse evicts whatever the block held
        self.ref[b] = 1
        return b

    def _forget(self, b):
        h = self.block_hash.pop(b, None)
        if h is not None and self.cached.get(h) == b:
            del self.cached[h]

    def free(self, b: int) -> None:
        self._check_block(b)
        if self.ref[b] <= 0:
            raise PoolError(f"block {b} is already free")
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free_queue.append(b)

    def incr_ref(self, b: int) -> None:
        self._check_block(b)
        if self.ref[b] <= 0:
            raise PoolError(f"block {b} is free")
        self.ref[b] += 1

    # -- sequences --------------------------------------------------------
    def _seq(self, sid):
        if sid not in self.seqs:
            raise BadIndex(f"unknown sequence {sid}")
        return self.seqs[sid]

    def seq_new(self) -> int:
        sid = self.next_seq
        self.next_seq += 1
        self.seqs[sid] = [[], 0]
        return sid

    def seq_fork(self, parent: int) -> int:
        blocks, n = self._seq(parent)
        for b in blocks:                     # all or nothing
            if self.ref[b] <= 0:
                raise PoolError(f"block {b} is free")
        for b in blocks:
            self.ref[b] += 1
        sid = self.seq_new()
        self.seqs[sid] = [list(blocks), n]
        return sid

    def seq_share_prefix(self, sid: int, blocks, num_tokens: int) -> None:
        """An empty sequence takes references on existing blocks holding its first
        num_tokens tokens (ceil(num_tokens / block_size) == len(blocks))."""
        seq = self._seq(sid)
        bs = self.block_size
        if seq[1] != 0 or len(blocks) != (num_tokens + bs - 1) // bs:
            raise InvalidArg("prefix must go into an empty sequence and fill its blocks")
        for b in blocks:
            self._check_block(b)
            if self.ref[b] <= 0:
                raise PoolError(f"block {b} is free")
        for b in blocks:
            self.ref[b] += 1
        seq[0] = list(blocks)
        seq[1] = num_tokens

    def seq_append(self, sid: int):
        """Room for one more token: returns (slot, cow_src, cow_dst), -1 when no copy."""
        blocks, n = self._seq(sid)
        bs = self.block_size
        src = dst = -1
        if n % bs == 0:
            blocks.append(self.alloc())
        else:
            last = blocks[-1]
            if self.ref[last] <= 1:
                self._forget(last)           # sole writer: the content changes
            if self.ref[last] > 1:
                new = self.alloc()
                self.ref[last] -= 1          # stays >= 1: the other holders keep it
                blocks[-1] = new
                src, dst = last, new
                self.cow_count += 1
        slot = blocks[-1] * bs + n % bs
        self.seqs[sid][1] = n + 1
        return slot, src, dst

    def seq_append_batch(self, sids):
        """seq_append on each of distinct sequences in order; all or nothing."""
        if len(set(sids)) != len(sids):
            raise InvalidArg("a sequence appears twice")
        need = 0
        for sid in sids:
            blocks, n = self._seq(sid)
            if n % self.block_size == 0 or self.ref[blocks[-1]] > 1:
                need += 1
        if need > len(self.free_queue):
            raise OutOfBlocks("not enough free blocks for the batch")
        slots, pairs = [], []
        for sid in sids:
            slot, src, dst = self.seq_append(sid)
            slots.append(slot)
            if src >= 0:
                pairs.append((src, dst))
        return slots, pairs

    def seq_free(self, sid: int) -> None:
        blocks, _ = self._seq(sid)
        for b, k in Counter(blocks).items():  # all or nothing
            if self.ref[b] < k:
                raise PoolError(f"block {b} has fewer references than the sequence holds")
        for b in blocks:
            self.free(b)
        del self.seqs[sid]

    def seq_len(self, sid: int) -> int:
        return self._seq(sid)[1]

    def seq_blocks(self, sid: int):
        return list(self._seq(sid)[0])

    # -- packing ----------------------------------------------------------
    def build_block_tables(self, sids, max_blocks: int):
        """Rows of physical ids padded with -1, plus the context lengths."""
        tables, lens = [], []
        for sid in sids:
            blocks, n = self._seq(sid)
            if len(blocks) > max_blocks:
                raise InvalidArg("table wider than max_blocks")
            tables.append(list(blocks) + [-1] * (max_blocks - len(blocks)))
            lens.append(n)
        return tables, lens

    # -- prefix cache -----------------------------------------------------
    def cache_block(self, b: int, h: int) -> bool:
        """Register full block ``b`` (in use) as holding content ``h``.  True
        when ``b`` is now the block for ``h``; False when another block holds it."""
        self._check_block(b)
        if self.ref[b] <= 0:
            raise PoolError(f"block {b} is free")
        if b in self.block_hash:
            if self.block_hash[b] != h:
                raise InvalidArg(f"block {b} already holds another hash")
            return True
        if h in self.cached:
            return False
        self.cached[h] = b
        self.block_hash[b] = h
        return True

    def cache_lookup(self, h: int) -> int:
        """The block holding ``h`` with one more reference taken, or -1."""
        b = self.cached.get(h, -1)
        if b < 0:
            return -1
        if self.ref[b] == 0:
            self.free_queue.remove(b)        # a freed block comes back to life
        self.ref[b] += 1
        self.cache_hits += 1
        return b

    def seq_match_prefix(self, sid: int, hashes) -> int:
        """An empty sequence takes the blocks of the leading hashes that hit."""
        blocks, n = self._seq(sid)
        if n != 0 or blocks:
            raise InvalidArg("a prefix can only be matched into an empty sequence")
        m = 0
        for h in hashes:
            b = self.cache_lookup(h)
            if b < 0:
                break
            blocks.append(b)
            m += 1
        self.seqs[sid][1] = m * self.block_size
        return m

    def stats(self):
        used = sum(1 for r in self.ref if r > 0)
        shared = sum(1 for r in self.ref if r > 1)
        return dict(num_blocks=self.num_blocks, free=len(self.free_queue), used=used,
                    shared=shared, cow_copies=self.cow_count, num_seqs=len(self.seqs),
                    cached=len(self.cached), cache_hits=self.cache_hits)
