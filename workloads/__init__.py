"""Seeded synthetic inputs for paged decode and prefill: the one module that both the oracle
side and the CUDA side of the tests (and bench.py) draw their inputs from.

It holds none of the method's arithmetic.  It only draws random numbers, casts
them to storage dtypes with torch's own conversions, and lays the results out
in the physical paged layout the method reads:

* key_cache / value_cache : [num_blocks, block_size, num_kv_heads, head_dim]
  ("PagedAttention 详解" §3, the FlashAttention-backend cache shape),
* block_tables            : [num_seqs, max_blocks] int32 physical block ids
  (same page, §10: a 100k-token table is 6250 int32 entries),
* context_lens            : [num_seqs] int32, counting the token appended this
  step (same page §4: append into the last block, then attend),
* slot_mapping            : [num_seqs] int64, slot = block * block_size + offset.

Poisoning (so that a kernel that reads what it must not read shows up as a NaN
or a wrong value instead of passing by luck):
* blocks no table references hold NaN codes,
* slots at or past position n-1 of each sequence hold NaN codes before the
  append (the append then fills n-1; n and beyond stay NaN),
* table entries past ceil(n / block_size) are -1.

The five workloads are the decode configurations this library is measured on;
``small_variant`` shrinks any of them for parity tests the oracle finishes in
seconds.  ``PREFILL_CONFIGS`` / ``make_prefill_inputs`` do the same for batches
of prefill chunks (new tokens appended through slot_mapping, then attended
causally over the cache).  Every draw comes from a seeded torch.Generator.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# storage dtypes by name -> (torch dtype, element bytes, NaN bit pattern)
_DT = {
    "f32": (torch.float32, 4),
    "f16": (torch.float16, 2),
    "bf16": (torch.bfloat16, 2),
    "fp8_e4m3": (torch.float8_e4m3fn, 1),
}
# one NaN encoding per storage dtype, as the raw integer of that width
_NAN_BITS = {"f32": 0x7FC00000, "f16": 0x7E00, "bf16": 0x7FC0, "fp8_e4m3": 0x7F}
_RAW = {4: torch.int32, 2: torch.int16, 1: torch.uint8}

E4M3_MAX = 448.0


def torch_dtype(name: str) -> torch.dtype:
    return _DT[name][0]


def elem_bytes(name: str) -> int:
    return _DT[name][1]


def raw_view(t: torch.Tensor, name: str) -> torch.Tensor:
    """Same storage viewed as unsigned-width integers (for bitwise compares)."""
    return t.view(_RAW[_DT[name][1]])


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    kv_dtype: str            # cache storage dtype
    q_dtype: str             # q / out dtype; also the dtype of the appended k, v
    ctx_lo: int              # context_len drawn uniform in [ctx_lo, ctx_hi]
    ctx_hi: int              # (context_len counts the appended token)
    fixed_lens: Optional[tuple] = None   # explicit context lens (overrides lo/hi)
    slack: float = 0.2       # extra free physical blocks, fraction of used
    fixed_num_blocks: Optional[int] = None
    prefix_tokens: int = 0   # shared-prefix tokens (whole blocks, same ids for all)
    suffix_lo: int = 0       # with a prefix: suffix length uniform in [lo, hi]
    suffix_hi: int = 0
    cow_last_block: bool = False   # last block shared with a parent -> COW on append
    partition: int = 0       # split-K tokens per partition the bench uses (0 = auto)
    fp8_scaled: bool = False

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


# The five decode workloads (sizes as stated for each).
CONFIGS = {
    1: DecodeConfig("tiny_paged_decode_fp32", 4, 4, 4, 64, 16, "f32", "f32", 0, 0,
                    fixed_lens=(17, 33, 64, 100), fixed_num_blocks=24, slack=0.0),
    2: DecodeConfig("llama2_7b_mha_fp16_b64", 64, 32, 32, 128, 16, "f16", "f16", 512, 2048,
                    partition=1024),
    3: DecodeConfig("llama3_8b_gqa_bf16_b128", 128, 32, 8, 128, 16, "bf16", "bf16", 1024, 8192),
    4: DecodeConfig("long_context_splitk_bf16_4x100k", 4, 32, 8, 128, 16, "bf16", "bf16", 0, 0,
                    fixed_lens=(100000,) * 4, partition=512, slack=0.02),
    5: DecodeConfig("prefix_shared_fp8_b256", 256, 32, 8, 128, 32, "fp8_e4m3", "bf16", 0, 0,
                    prefix_tokens=1024, suffix_lo=64, suffix_hi=512, cow_last_block=True,
                    fp8_scaled=True),
}


# the same workloads by name
DECODE_WORKLOADS = {cfg.name: cfg for cfg in CONFIGS.values()}


def small_variant(cfg: DecodeConfig, num_seqs: int, ctx_lo: int, ctx_hi: int,
                  prefix_tokens: Optional[int] = None) -> DecodeConfig:
    """Same heads / dims / dtypes / structure, fewer and shorter sequences."""
    kw = dict(num_seqs=num_seqs, fixed_lens=None, fixed_num_blocks=None,
              name=cfg.name + f"_small{num_seqs}")
    if cfg.prefix_tokens:
        p = cfg.prefix_tokens if prefix_tokens is None else prefix_tokens
        kw.update(prefix_tokens=p, suffix_lo=ctx_lo, suffix_hi=ctx_hi)
    else:
        kw.update(ctx_lo=ctx_lo, ctx_hi=ctx_hi)
    return dataclasses.replace(cfg, **kw)


@dataclasses.dataclass
class DecodeInputs:
    cfg: DecodeConfig
    q: torch.Tensor                 # [S, Hq, D] q_dtype
    key_cache: torch.Tensor         # [NB, bs, Hkv, D] kv_dtype, state before this step
    value_cache: torch.Tensor
    key_new: torch.Tensor           # [S, Hkv, D] q_dtype: this step's k, v
    value_new: torch.Tensor
    slot_mapping: torch.Tensor      # [S] int64, slot of the appended token
    block_tables: torch.Tensor      # [S, MB] int32 after any copy-on-write
    block_tables_pre: torch.Tensor  # [S, MB] int32 before copy-on-write
    context_lens: torch.Tensor      # [S] int32, including the appended token
    copy_pairs: torch.Tensor        # [n, 2] int32 (src, dst), host; empty without COW
    k_scale: float
    v_scale: float
    scale: float
    num_blocks: int
    max_blocks: int
    free_blocks: torch.Tensor       # physical ids referenced by no table

    @property
    def max_ctx(self) -> int:
        return int(self.context_lens.max().item()) if self.context_lens.numel() else 0


def _draw_lens(cfg: DecodeConfig, g: torch.Generator) -> torch.Tensor:
    if cfg.fixed_lens is not None:
        assert len(cfg.fixed_lens) == cfg.num_seqs
        return torch.tensor(cfg.fixed_lens, dtype=torch.int64)
    if cfg.prefix_tokens:
        suf = torch.randint(cfg.suffix_lo, cfg.suffix_hi + 1, (cfg.num_seqs,), generator=g)
        return suf + cfg.prefix_tokens
    return torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (cfg.num_seqs,), generator=g)


def draw_context_lens(cfg: DecodeConfig, seed: int) -> torch.Tensor:
    """The context lengths make_decode_inputs(cfg, seed) draws (int64 [S])."""
    return _draw_lens(cfg, torch.Generator(device="cpu").manual_seed(seed))


def _fill_normal(t: torch.Tensor, dtype_name: str, g: torch.Generator,
                 scale_div: float = 1.0, chunk: int = 1 << 26) -> None:
    """Fill t (any shape) with N(0,1) draws cast to its dtype, chunked to bound memory.
    For fp8 the draw is divided by scale_div and clamped to the e4m3 range first."""
    flat = t.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        x = torch.randn(m, generator=g, device=t.device, dtype=torch.float32)
        if dtype_name == "fp8_e4m3":
            x = (x / scale_div).clamp_(-E4M3_MAX, E4M3_MAX)
        flat[i:i + m] = x.to(t.dtype)


def _amax_normal(n: int, g: torch.Generator, device, chunk: int = 1 << 26) -> float:
    """amax |x| over n N(0,1) draws, consuming the generator exactly as _fill_normal would."""
    a = 0.0
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        x = torch.randn(m, generator=g, device=device, dtype=torch.float32)
        a = max(a, float(x.abs().max().item()))
    return a


def make_decode_inputs(cfg: DecodeConfig, seed: int, device="cpu") -> DecodeInputs:
    """Seeded inputs for one decode step of ``cfg`` on ``device``.

    Structure: every sequence owns ceil(n/bs) logical blocks mapped to shuffled
    physical ids; with a prefix, the first prefix_tokens/bs entries of every
    table are the same physical ids; with cow_last_block, the block that will
    receive the appended token is a shared block (a parent also holds it), so
    the step first copies it to a fresh block (copy_pairs) and the post-COW
    table points there.  When the appended token opens a new block, that block
    is fresh and no copy is needed.
    """
    S, Hkv, D, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    gh = torch.Generator(device="cpu").manual_seed(seed)
    lens = _draw_lens(cfg, gh)
    nblk = (lens + bs - 1) // bs                       # blocks after the append
    MB = int(nblk.max().item()) if S else 1
    prefix_blocks = cfg.prefix_tokens // bs
    assert cfg.prefix_tokens % bs == 0

    # physical ids needed: shared prefix + private blocks (+ parent-held shared last block)
    priv = nblk - prefix_blocks                        # private logical blocks per seq
    cow = torch.zeros(S, dtype=torch.bool)
    if cfg.cow_last_block:
        cow = ((lens - 1) % bs) != 0                   # append lands inside an existing block
    used = prefix_blocks + int(priv.sum().item()) + int(cow.sum().item())
    NB = cfg.fixed_num_blocks or int(math.ceil(used * (1.0 + cfg.slack)))
    NB = max(NB, used)
    perm = torch.randperm(NB, generator=gh).to(torch.int32)

    tables = torch.full((S, MB), -1, dtype=torch.int32)
    tables_pre = torch.full((S, MB), -1, dtype=torch.int32)
    pairs = []
    cur = 0
    prefix_ids = perm[cur:cur + prefix_blocks]
    cur += prefix_blocks
    for s in range(S):
        k = int(priv[s])
        ids = perm[cur:cur + k]
        cur += k
        row = torch.cat([prefix_ids, ids])
        tables[s, :row.numel()] = row
        tables_pre[s, :row.numel()] = row
        if cow[s]:
            src = int(perm[cur])
            cur += 1
            last = int(nblk[s]) - 1
            tables_pre[s, last] = src
            pairs.append((src, int(tables[s, last])))
    referenced = perm[:cur]
    free_ids = perm[cur:]

    dev = torch.device(device)
    gd = torch.Generator(device=dev).manual_seed(seed + 1000003)
    kv_t = torch_dtype(cfg.kv_dtype)
    q_t = torch_dtype(cfg.q_dtype)
    shape = (NB, bs, Hkv, D)
    kc = torch.empty(shape, dtype=kv_t, device=dev)
    vc = torch.empty(shape, dtype=kv_t, device=dev)

    k_scale = v_scale = 1.0
    if cfg.fp8_scaled:
        # per-tensor scales: amax of the fp32 draws over the whole cache / e4m3 max;
        # the same draws (same generator state) then fill the cache.
        st = gd.get_state()
        k_scale = _amax_normal(kc.numel(), gd, dev) / E4M3_MAX
        v_scale = _amax_normal(vc.numel(), gd, dev) / E4M3_MAX
        gd.set_state(st)
    _fill_normal(kc, cfg.kv_dtype, gd, k_scale)
    _fill_normal(vc, cfg.kv_dtype, gd, v_scale)

    q = torch.empty((S, cfg.num_q_heads, D), dtype=q_t, device=dev)
    _fill_normal(q, cfg.q_dtype, gd)
    key_new = torch.empty((S, Hkv, D), dtype=q_t, device=dev)
    value_new = torch.empty((S, Hkv, D), dtype=q_t, device=dev)
    _fill_normal(key_new, cfg.q_dtype, gd)
    _fill_normal(value_new, cfg.q_dtype, gd)

    # ---- poisoning -------------------------------------------------------
    nan = _NAN_BITS[cfg.kv_dtype]
    rk, rv = raw_view(kc, cfg.kv_dtype), raw_view(vc, cfg.kv_dtype)
    nan_t = torch.tensor(nan, dtype=rk.dtype, device=dev)  # every pattern fits the signed width
    if free_ids.numel():
        fi = free_ids.to(dev, torch.int64)
        rk[fi] = nan_t
        rv[fi] = nan_t
    # fresh COW destinations hold garbage until the copy
    if pairs:
        di = torch.tensor([p[1] for p in pairs], dtype=torch.int64, device=dev)
        rk[di] = nan_t
        rv[di] = nan_t
    # slots at/after position n-1 in each sequence's pre-step view
    pb, po = [], []
    for s in range(S):
        n = int(lens[s])
        for pos in range(max(n - 1, 0), int(nblk[s]) * bs):
            pb.append(int(tables_pre[s, pos // bs]))
            po.append(pos % bs)
    if pb:
        bi = torch.tensor(pb, dtype=torch.int64, device=dev)
        oi = torch.tensor(po, dtype=torch.int64, device=dev)
        rk[bi, oi] = nan_t
        rv[bi, oi] = nan_t

    slots = torch.empty(S, dtype=torch.int64)
    for s in range(S):
        n = int(lens[s])
        pos = n - 1
        slots[s] = int(tables[s, pos // bs]) * bs + pos % bs if n > 0 else -1

    return DecodeInputs(
        cfg=cfg, q=q, key_cache=kc, value_cache=vc, key_new=key_new, value_new=value_new,
        slot_mapping=slots.to(dev), block_tables=tables.to(dev),
        block_tables_pre=tables_pre.to(dev), context_lens=lens.to(torch.int32).to(dev),
        copy_pairs=torch.tensor(pairs, dtype=torch.int32).reshape(-1, 2),
        k_scale=float(k_scale), v_scale=float(v_scale), scale=cfg.scale,
        num_blocks=NB, max_blocks=MB, free_blocks=free_ids.clone())


def kv_bytes_per_token(cfg: DecodeConfig) -> int:
    """K plus V bytes one token of one sequence occupies (all kv heads)."""
    return 2 * cfg.num_kv_heads * cfg.head_dim * elem_bytes(cfg.kv_dtype)


# --------------------------------------------------------------------- prefill

@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    """A batch of prefill chunks: sequence s already holds c_s cached tokens and
    this step appends L_s new ones (their K, V through slot_mapping), then the
    new tokens attend causally over all c_s + L_s."""
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str               # q / out / cache dtype (f16 or bf16)
    q_lo: int                # L_s uniform in [q_lo, q_hi]
    q_hi: int
    ctx_lo: int              # c_s uniform in [ctx_lo, ctx_hi]
    ctx_hi: int
    fixed_q: Optional[tuple] = None
    fixed_ctx: Optional[tuple] = None
    slack: float = 0.1

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


PREFILL_CONFIGS = {
    # Llama-3-8B attention shapes, chunked prefill: 16 chunks of 2048 new tokens
    # on top of 0..6144 cached tokens each.
    "llama3_8b_gqa_bf16_chunked_prefill": PrefillConfig(
        "llama3_8b_gqa_bf16_chunked_prefill", 16, 32, 8, 128, 16, "bf16", 2048, 2048, 0, 6144),
    # the same shapes, prefill from an empty cache: 8 prompts of 1024..4096 tokens
    "llama3_8b_gqa_bf16_prefill": PrefillConfig(
        "llama3_8b_gqa_bf16_prefill", 8, 32, 8, 128, 16, "bf16", 1024, 4096, 0, 0),
}


@dataclasses.dataclass
class PrefillInputs:
    cfg: PrefillConfig
    q: torch.Tensor                 # [T, Hq, D]
    key_cache: torch.Tensor         # [NB, bs, Hkv, D], state before this step's append
    value_cache: torch.Tensor
    key_new: torch.Tensor           # [T, Hkv, D]: the new tokens' k, v
    value_new: torch.Tensor
    slot_mapping: torch.Tensor      # [T] int64
    block_tables: torch.Tensor      # [S, MB] int32
    context_lens: torch.Tensor      # [S] int32: c_s + L_s
    query_start: torch.Tensor       # [S + 1] int32
    cached_lens: torch.Tensor       # [S] int64: c_s
    scale: float
    num_blocks: int
    max_blocks: int

    @property
    def max_query_len(self) -> int:
        qs = self.query_start.cpu()
        return int((qs[1:] - qs[:-1]).max().item()) if qs.numel() > 1 else 0

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1].item())


def make_prefill_inputs(cfg: PrefillConfig, seed: int, device="cpu") -> PrefillInputs:
    """Seeded inputs for one prefill step of ``cfg`` on ``device``.

    Every sequence owns ceil((c + L) / bs) shuffled physical blocks.  Cached
    positions hold N(0,1) draws; positions c..end of the last block, blocks no
    table references and this step's slots before the append hold NaN codes;
    table entries past the sequence's blocks are -1.
    """
    S, Hkv, D, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    gh = torch.Generator(device="cpu").manual_seed(seed)
    if cfg.fixed_q is not None:
        L = torch.tensor(cfg.fixed_q, dtype=torch.int64)
    else:
        L = torch.randint(cfg.q_lo, cfg.q_hi + 1, (S,), generator=gh)
    if cfg.fixed_ctx is not None:
        c = torch.tensor(cfg.fixed_ctx, dtype=torch.int64)
    else:
        c = torch.randint(cfg.ctx_lo, cfg.ctx_hi + 1, (S,), generator=gh)
    n = c + L
    nblk = (n + bs - 1) // bs
    MB = max(int(nblk.max().item()) if S else 1, 1)
    used = int(nblk.sum().item())
    NB = max(int(math.ceil(used * (1.0 + cfg.slack))), used, 1)
    perm = torch.randperm(NB, generator=gh).to(torch.int32)
    tables = torch.full((S, MB), -1, dtype=torch.int32)
    cur = 0
    for s in range(S):
        k = int(nblk[s])
        tables[s, :k] = perm[cur:cur + k]
        cur += k
    free_ids = perm[cur:]

    dev = torch.device(device)
    gd = torch.Generator(device=dev).manual_seed(seed + 7919)
    t = torch_dtype(cfg.dtype)
    kc = torch.empty((NB, bs, Hkv, D), dtype=t, device=dev)
    vc = torch.empty_like(kc)
    _fill_normal(kc, cfg.dtype, gd)
    _fill_normal(vc, cfg.dtype, gd)
    T = int(L.sum().item())
    q = torch.empty((T, cfg.num_q_heads, D), dtype=t, device=dev)
    kn = torch.empty((T, Hkv, D), dtype=t, device=dev)
    vn = torch.empty_like(kn)
    _fill_normal(q, cfg.dtype, gd)
    _fill_normal(kn, cfg.dtype, gd)
    _fill_normal(vn, cfg.dtype, gd)

    nan_t = torch.tensor(_NAN_BITS[cfg.dtype], dtype=_RAW[_DT[cfg.dtype][1]], device=dev)
    rk, rv = raw_view(kc, cfg.dtype), raw_view(vc, cfg.dtype)
    if free_ids.numel():
        fi = free_ids.to(dev, torch.int64)
        rk[fi] = nan_t
        rv[fi] = nan_t
    pb, po, slots = [], [], []
    for s in range(S):
        for pos in range(int(c[s]), int(nblk[s]) * bs):
            pb.append(int(tables[s, pos // bs]))
            po.append(pos % bs)
        for pos in range(int(c[s]), int(n[s])):
            slots.append(int(tables[s, pos // bs]) * bs + pos % bs)
    if pb:
        bi = torch.tensor(pb, dtype=torch.int64, device=dev)
        oi = torch.tensor(po, dtype=torch.int64, device=dev)
        rk[bi, oi] = nan_t
        rv[bi, oi] = nan_t
    qs = torch.zeros(S + 1, dtype=torch.int32)
    qs[1:] = torch.cumsum(L, 0).to(torch.int32)
    return PrefillInputs(
        cfg=cfg, q=q, key_cache=kc, value_cache=vc, key_new=kn, value_new=vn,
        slot_mapping=torch.tensor(slots, dtype=torch.int64).to(dev),
        block_tables=tables.to(dev), context_lens=n.to(torch.int32).to(dev),
        query_start=qs.to(dev), cached_lens=c, scale=cfg.scale, num_blocks=NB, max_blocks=MB)


def prefill_flops(cfg: PrefillConfig, query_start: torch.Tensor, context_lens: torch.Tensor) -> int:
    """Multiply-adds x 2 of the causal attention the step must do: each new token
    at position p scores p + 1 keys (Q.K) and sums p + 1 values (P.V)."""
    qs = query_start.cpu().to(torch.int64)
    n = context_lens.cpu().to(torch.int64)
    L = qs[1:] - qs[:-1]
    c = n - L
    keys = int((L * c + L * (L + 1) // 2).sum().item())    # sum over new tokens of p + 1
    return 4 * keys * cfg.num_q_heads * cfg.head_dim
