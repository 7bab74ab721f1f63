"""Seeded synthetic decode steps shaped like the paged-attention workloads.

Shared by the tests, the benchmark and the oracle's callers; it holds none of
the method's arithmetic (no attention, no scatter, no copy).  It draws context
lengths, builds block tables / slot mappings / copy-on-write pairs with the
host block manager, and fills pools with seeded random numbers.

A ``DecodeStep`` is the state *before* one decode step of one layer:
  1. ``copy_pairs``: copy-on-write block copies planned for this step,
  2. ``new_key`` / ``new_value`` written to ``slot_mapping`` (one token per
     live sequence, -1 for empty sequences),
  3. decode attention of ``q`` over ``context_lens`` tokens, which include the
     token written in 2.

Workloads (sizes as named by their builders):
  * ``tiny``          -- 4 seqs, context lens [7, 16, 33, 100], 4 q = 4 kv heads,
                         head_dim 64, fp32, 64-block pool, block_size 16 or 4.
  * ``llama7b``       -- 64 seqs, 32 = 32 heads, head_dim 128, bf16, block_size 16,
                         context lens uniform [128, 2048], 8192-block shuffled pool.
  * ``gqa``           -- 256 seqs, 32 q / 8 kv heads, bf16, log-normal context lens
                         (median 1000, sigma 1.0, capped 8192), 90 % occupied pool.
  * ``shared_prefix`` -- 16 prompts x 8 samples sharing the prompt's blocks,
                         per-sample suffix uniform [0, suffix_max], 32 q / 8 kv heads.
  * ``long_context``  -- 8 seqs, context lens uniform [32768, 131072], 64 q / 8 kv
                         heads, block_size 8 / 16 / 32, partitions of 512 tokens.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence as Seq, Tuple

import numpy as np
import torch

from .blocks import BlockManager, BlockPool, Sequence, block_table_array

ELEMENT_BYTES = {torch.float32: 4, torch.bfloat16: 2}


@dataclass
class DecodeStep:
    name: str
    dtype: torch.dtype
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray          # int32 [S]; includes this step's token
    block_tables: np.ndarray          # int32 [S][max_blocks]; -1 past the end
    scale: float
    partition_size: int
    q: torch.Tensor                   # [S][Hq][d]
    k_cache: torch.Tensor             # [NB][Hkv][B][d], before this step's copies/writes
    v_cache: torch.Tensor
    new_key: torch.Tensor             # [T][Hkv][d]
    new_value: torch.Tensor
    slot_mapping: np.ndarray          # int64 [T]; -1 = no write
    copy_pairs: np.ndarray            # int64 [n][2] (src, dst)
    meta: Dict = field(default_factory=dict)
    query_start: Optional[np.ndarray] = None   # prefill: int32 [S + 1]; q / new K,V hold every new token

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def element_bytes(self) -> int:
        return ELEMENT_BYTES[self.dtype]

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0


def algorithmic_bytes(step: DecodeStep, unique: bool = True) -> int:
    """Bytes the decode of one layer must move: every valid token's K and V
    gathered once through the block table ("PagedAttention blog" section 3(3)),
    the query read and the output written, and the table entries and lengths
    that locate them:

        sum_s ctx_s * Hkv * d * 2 * e      K and V of valid tokens
      + 2 * S * Hq * d * e                 q read, out written
      + sum_s ceil(ctx_s / B) * 4 + 4 * S  block-table entries and context lens

    With ``unique`` the K/V of a physical block shared by several sequences
    are counted once (for each shared block, the most tokens any sharer reads
    from it); otherwise per sequence ("logical" bytes).
    """
    e = step.element_bytes
    Hkv, d, B = step.num_kv_heads, step.head_dim, step.block_size
    ctx = step.context_lens.astype(np.int64)
    if unique:
        tokens_in_block: Dict[int, int] = {}
        for s in range(step.num_seqs):
            c = int(ctx[s])
            for i in range(-(-c // B)):
                blk = int(step.block_tables[s, i])
                n = min(B, c - i * B)
                tokens_in_block[blk] = max(tokens_in_block.get(blk, 0), n)
        kv_tokens = sum(tokens_in_block.values())
    else:
        kv_tokens = int(ctx.sum())
    kv = kv_tokens * Hkv * d * 2 * e
    qo = 2 * step.num_seqs * step.num_heads * d * e
    tables = int(sum(-(-int(c) // B) for c in ctx)) * 4 + 4 * step.num_seqs
    return int(kv + qo + tables)


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, dtype, device, gen) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32 if dtype == torch.float32 else dtype, device=device)
    t.normal_(generator=gen)
    return t


def _build(name: str, *, dtype, num_heads: int, num_kv_heads: int, head_dim: int,
           block_size: int, num_blocks: int, free_order, groups: List[Tuple[int, List[int]]],
           seed: int, device, poison: bool, partition_size: int,
           meta: Optional[Dict] = None) -> DecodeStep:
    """Common builder.

    ``groups``: list of (prompt_len, [history suffix length per sample]).  A
    group with one sample and prompt_len = ctx - 1 is an independent sequence.
    All samples of a group share the prompt's physical blocks.  Every sample
    then appends one token for this step, except in a group whose prompt_len
    is negative: that is one empty sequence (context 0) with no write.
    """
    pool = BlockPool(num_blocks, free_order)
    mgr = BlockManager(pool, block_size)
    seqs: List[Sequence] = []
    history_copies: List[Tuple[int, int, int]] = []   # (src, dst, slots filled at copy time)
    step_slots: List[int] = []
    step_copies: List[Tuple[int, int]] = []
    live: List[bool] = []
    for prompt_len, suffixes in groups:
        base = mgr.new_sequence()
        mgr.append_tokens(base, max(prompt_len, 0))
        members = [base] + [mgr.fork(base) for _ in range(len(suffixes) - 1)]
        # history: samples generate their suffix tokens round-robin
        for t in range(max(suffixes) if suffixes else 0):
            for m, L in zip(members, suffixes):
                if t < L:
                    pos = m.num_tokens
                    _, cps = mgr.append_tokens(m, 1)
                    for src, dst in cps:
                        history_copies.append((src, dst, pos % block_size))
        seqs.extend(members)
        live.extend([prompt_len >= 0] * len(members))
    for m, is_live in zip(seqs, live):
        if not is_live:
            step_slots.append(-1)
            continue
        slots, cps = mgr.append_tokens(m, 1)
        step_slots.extend(slots)
        step_copies.extend(cps)

    S = len(seqs)
    ctx = np.array([m.num_tokens for m in seqs], dtype=np.int32)
    tables = block_table_array(seqs)
    Hkv, d, B = num_kv_heads, head_dim, block_size

    gen = _generator(device, seed)
    k_cache = _normal((num_blocks, Hkv, B, d), dtype, device, gen)
    v_cache = _normal((num_blocks, Hkv, B, d), dtype, device, gen)
    # history copy-on-write: the copy keeps the source's filled slots; the
    # slots the sample wrote afterwards keep their own (already random) values.
    for src, dst, filled in history_copies:
        if filled:
            k_cache[dst, :, :filled] = k_cache[src, :, :filled]
            v_cache[dst, :, :filled] = v_cache[src, :, :filled]
    q = _normal((S, num_heads, d), dtype, device, gen)
    T = len(step_slots)
    new_key = _normal((T, Hkv, d), dtype, device, gen)
    new_value = _normal((T, Hkv, d), dtype, device, gen)

    if poison:
        # every slot that holds no token before this step becomes NaN:
        # free blocks, reservation slots, and the slots this step will write.
        used = np.zeros((num_blocks, B), dtype=bool)
        for m, c in zip(seqs, ctx):
            before = int(c) - 1 if int(c) > 0 else 0
            for i, blk in enumerate(m.block_table):
                n = min(B, max(0, before - i * B))
                used[blk, :n] = True
        # blocks that are a copy destination this step hold nothing yet
        for _, dst in step_copies:
            used[dst, :] = False
        mask = torch.from_numpy(~used).to(device)
        nan = float("nan")
        k_cache.masked_fill_(mask[:, None, :, None], nan)
        v_cache.masked_fill_(mask[:, None, :, None], nan)

    info = dict(meta or {})
    info.update(num_history_copies=len(history_copies))
    return DecodeStep(
        name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=Hkv, head_dim=d,
        block_size=B, num_blocks=num_blocks, context_lens=ctx, block_tables=tables,
        scale=float(np.float32(1.0 / math.sqrt(d))), partition_size=partition_size,
        q=q, k_cache=k_cache, v_cache=v_cache, new_key=new_key, new_value=new_value,
        slot_mapping=np.array(step_slots, dtype=np.int64),
        copy_pairs=np.array(step_copies, dtype=np.int64).reshape(-1, 2), meta=info)


def independent(name: str, context_lens: Seq[int], *, dtype=torch.bfloat16, num_heads=8,
                num_kv_heads=8, head_dim=128, block_size=16, num_blocks=None,
                occupancy: float = 0.9, seed=0, device="cpu", poison=False,
                partition_size=512, shuffle=True, meta=None) -> DecodeStep:
    """Independent sequences with the given context lengths (this step's token included)."""
    ctx = [int(c) for c in context_lens]
    used = sum(-(-c // block_size) for c in ctx)
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(used / occupancy)))
    rng = np.random.default_rng(seed + 7919)
    order = rng.permutation(num_blocks) if shuffle else np.arange(num_blocks)
    groups = [(c - 1, [0]) for c in ctx]   # ctx 0 -> prompt_len -1: an empty sequence
    return _build(name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                  head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
                  free_order=order, groups=groups, seed=seed, device=device, poison=poison,
                  partition_size=partition_size, meta=meta)


def tiny(block_size: int = 16, seed: int = 0, device="cpu", poison=False,
         partition_size: int = 512) -> DecodeStep:
    """4 seqs, context lens [7, 16, 33, 100], 4 = 4 heads, d 64, fp32, 64-block pool;
    physical ids are the first blocks of a seeded permutation of 0..63, in logical order."""
    return independent(f"tiny_fp32_b{block_size}", [7, 16, 33, 100], dtype=torch.float32,
                       num_heads=4, num_kv_heads=4, head_dim=64, block_size=block_size,
                       num_blocks=64, seed=seed, device=device, poison=poison,
                       partition_size=partition_size)


def llama7b(seed: int = 0, device="cpu", poison=False, partition_size: int = 512) -> DecodeStep:
    """Llama-7B-like decode layer: 64 seqs, 32 = 32 heads, d 128, bf16, block 16,
    context lens uniform [128, 2048], blocks popped from a shuffled 8192-block free list."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(128, 2048, size=64, endpoint=True)
    return independent("llama7b_bf16", ctx, dtype=torch.bfloat16, num_heads=32, num_kv_heads=32,
                       head_dim=128, block_size=16, num_blocks=8192, seed=seed, device=device,
                       poison=poison, partition_size=partition_size)


def gqa(seed: int = 0, sigma: float = 1.0, device="cpu", poison=False,
        partition_size: int = 512, num_seqs: int = 256) -> DecodeStep:
    """GQA decode: 256 seqs, 32 q / 8 kv heads, d 128, bf16, block 16, context lens
    log-normal (median 1000, sigma as given, capped to [1, 8192]), pool 90 % occupied."""
    rng = np.random.default_rng(seed)
    ctx = np.clip(np.round(np.exp(math.log(1000.0) + sigma * rng.standard_normal(num_seqs))), 1, 8192)
    return independent(f"gqa_bf16_sigma{sigma:g}", ctx.astype(np.int64), dtype=torch.bfloat16,
                       num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, occupancy=0.9,
                       seed=seed, device=device, poison=poison, partition_size=partition_size,
                       meta=dict(sigma=sigma))


def shared_prefix(seed: int = 0, prompt_len: int = 512, suffix_max: int = 512, prompts: int = 16,
                  samples: int = 8, device="cpu", poison=False, partition_size: int = 512,
                  num_heads: int = 32, num_kv_heads: int = 8, head_dim: int = 128,
                  block_size: int = 16) -> DecodeStep:
    """Parallel sampling: ``prompts`` prompts x ``samples`` samples sharing the prompt's
    blocks (ref count = samples), per-sample suffix uniform [0, suffix_max] in private
    blocks; 32 q / 8 kv heads, d 128, bf16, block 16.  A partial last prompt block is
    copied on write by each sharer that writes into it while it is still shared."""
    rng = np.random.default_rng(seed)
    groups = [(prompt_len, [int(x) for x in rng.integers(0, suffix_max, size=samples, endpoint=True)])
              for _ in range(prompts)]
    B = block_size
    per_seq = [prompt_len + max(sfx) + 1 for _, sfx in groups]
    worst = prompts * (-(-prompt_len // B)) + sum(samples * (-(-(max(sfx) + 2) // B) + 1)
                                                  for _, sfx in groups)
    num_blocks = int(math.ceil(worst / 0.9))
    order = np.random.default_rng(seed + 7919).permutation(num_blocks)
    del per_seq
    return _build(f"shared_prefix_p{prompt_len}_bf16", dtype=torch.bfloat16, num_heads=num_heads,
                  num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=B, num_blocks=num_blocks,
                  free_order=order, groups=groups, seed=seed, device=device, poison=poison,
                  partition_size=partition_size,
                  meta=dict(prompts=prompts, samples=samples, prompt_len=prompt_len,
                            suffix_max=suffix_max))


def long_context(seed: int = 0, block_size: int = 16, device="cpu", poison=False,
                 partition_size: int = 512, num_seqs: int = 8) -> DecodeStep:
    """Long-context decode: 8 seqs, context lens uniform [32768, 131072] (the same draw
    for every block size), 64 q / 8 kv heads, d 128, bf16, pool = 1.1 x used, shuffled."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(32768, 131072, size=num_seqs, endpoint=True)
    return independent(f"long_context_b{block_size}_bf16", ctx, dtype=torch.bfloat16, num_heads=64,
                       num_kv_heads=8, head_dim=128, block_size=block_size, occupancy=1 / 1.1,
                       seed=seed, device=device, poison=poison, partition_size=partition_size)


def prefill_chunk(seed: int = 0, num_seqs: int = 16, cached: int = 1024, new: int = 256, device="cpu",
                  num_heads: int = 32, num_kv_heads: int = 8, head_dim: int = 128, block_size: int = 16,
                  partition_size: int = 512, dtype=torch.bfloat16) -> DecodeStep:
    """Chunked prefill: each sequence holds ``cached`` tokens and appends ``new``
    tokens whose K/V are written this step and whose queries attend causally."""
    used = num_seqs * (-(-(cached + new) // block_size))
    num_blocks = int(math.ceil(used / 0.9))
    order = np.random.default_rng(seed + 7919).permutation(num_blocks)
    pool = BlockPool(num_blocks, order)
    mgr = BlockManager(pool, block_size)
    seqs, slots = [], []
    for _ in range(num_seqs):
        sq = mgr.new_sequence()
        mgr.append_tokens(sq, cached)
        sl, _ = mgr.append_tokens(sq, new)
        slots.extend(sl)
        seqs.append(sq)
    gen = _generator(device, seed)
    Hkv, d, B = num_kv_heads, head_dim, block_size
    k_cache = _normal((num_blocks, Hkv, B, d), dtype, device, gen)
    v_cache = _normal((num_blocks, Hkv, B, d), dtype, device, gen)
    T = num_seqs * new
    q = _normal((T, num_heads, d), dtype, device, gen)
    new_key = _normal((T, Hkv, d), dtype, device, gen)
    new_value = _normal((T, Hkv, d), dtype, device, gen)
    return DecodeStep(
        name=f"prefill_{cached}+{new}", dtype=dtype, num_heads=num_heads, num_kv_heads=Hkv, head_dim=d,
        block_size=B, num_blocks=num_blocks,
        context_lens=np.array([sq.num_tokens for sq in seqs], dtype=np.int32),
        block_tables=block_table_array(seqs), scale=float(np.float32(1.0 / math.sqrt(d))),
        partition_size=partition_size, q=q, k_cache=k_cache, v_cache=v_cache, new_key=new_key,
        new_value=new_value, slot_mapping=np.array(slots, dtype=np.int64),
        copy_pairs=np.zeros((0, 2), dtype=np.int64), meta=dict(cached=cached, new=new),
        query_start=np.arange(0, T + 1, new, dtype=np.int32))


def prefill_flops(step: DecodeStep) -> int:
    """Useful multiply-adds x 2 of a prefill step: q.K and p.V of every new token over
    the positions it sees, 4 * d * Hq * (pos + 1) each."""
    total = 0
    qs = step.query_start
    for s in range(step.num_seqs):
        n = int(qs[s + 1] - qs[s])
        c = int(step.context_lens[s])
        # positions c-n .. c-1, each seeing pos + 1 tokens
        total += sum(range(c - n + 1, c + 1))
    return 4 * step.head_dim * step.num_heads * total


def prefill_tc_mma_flops(step: DecodeStep, rows: int = 128, tile: int = 32) -> int:
    """Tensor-core flops the tcgen05 prefill issues: per tile of 128 query rows x
    32 tokens, S = Q.K^T (2*128*32*d) and P.V with P as hi + lo (2 x 2*128*32*d),
    for every tile a query block reaches (masked positions and padding rows
    included)."""
    g = step.num_heads // step.num_kv_heads
    tq = rows // g
    tiles = 0
    qs = step.query_start
    for s in range(step.num_seqs):
        n = int(qs[s + 1] - qs[s])
        c = int(step.context_lens[s])
        for qb in range(-(-n // tq)):
            pos_max = c - n + min(n, (qb + 1) * tq) - 1
            if pos_max >= 0:
                tiles += pos_max // tile + 1
    return tiles * step.num_kv_heads * 3 * 2 * rows * tile * step.head_dim


WORKLOADS = {
    "tiny": tiny,
    "llama7b": llama7b,
    "gqa": gqa,
    "shared_prefix": shared_prefix,
    "long_context": long_context,
    "prefill_chunk": prefill_chunk,
}
