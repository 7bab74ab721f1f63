"""fp64 oracle: scatter into a paged KV pool, copy-on-write block copy, and
decode attention through a per-sequence block table.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain, slow and
written to be checked by eye against the pages:

* A sequence's tokens are cut into logical blocks of ``B`` tokens; logical
  block ``i`` holds tokens ``[i*B, (i+1)*B)``.  The block table maps logical
  block ``i`` to a physical block of a shared pool.  The last logical block may
  be partly filled; its unused slots are the "reservation" and hold nothing.
  ("PagedAttention blog", section 3(3), prefill step.)
* At decode time attention is computed as if the tokens were contiguous; the
  data are fetched from the physical blocks through the block table.
  ("PagedAttention blog", section 3(3), decode step; "Month 2 ·
  PagedAttention", section 06: the kernel is ordinary attention that can
  gather K and V from non-contiguous addresses.)
* ``slot_mapping`` says where each new token's K/V is written
  ("Month 2 · PagedAttention", section 03, reading 4).  Reading adopted
  (the pages do not write it out): slot = physical_block * B + offset, so
  block = slot // B and offset = slot % B; a negative slot means "no write".
* Copy-on-write: when a sharer writes into a physical block whose reference
  count is above one, a new physical block is taken and the old block's
  contents are copied into it ("PagedAttention blog", section 4, step 2).
  Reading adopted: the whole block is copied, unfilled slots included.

Pool layout (the pages fix none): ``cache[num_blocks][num_kv_heads][B][d]``.
Query heads ``[kvh*g, (kvh+1)*g)`` share kv head ``kvh`` (g = Hq / Hkv); the
pages are silent on grouped-query attention, this is the contiguous grouping.
Attention formula (the pages print none): softmax(scale * q . K^T) . V over
all ``context_len`` tokens of the sequence, the token written this step
included, no causal mask inside a decode step.
"""

from __future__ import annotations

import numpy as np


def gather_kv(cache, block_table, context_len, kv_head):
    """Rows 0..context_len-1 of one kv head, read through the block table.

    ``cache``: [num_blocks][Hkv][B][d]; ``block_table``: physical block id of
    each logical block.  Entries past ceil(context_len / B) are never read, and
    slots past ``context_len`` in the last block (the reservation) are dropped.
    """
    block_size = cache.shape[2]
    head_dim = cache.shape[3]
    n_logical = -(-int(context_len) // block_size)
    pieces = []
    for i in range(n_logical):
        physical = int(block_table[i])
        pieces.append(np.asarray(cache[physical, kv_head], dtype=np.float64))
    if not pieces:
        return np.zeros((0, head_dim), dtype=np.float64)
    return np.concatenate(pieces, axis=0)[: int(context_len)]


def decode_attention_one(q_head, k_rows, v_rows, scale):
    """Ordinary attention of one query vector against contiguous rows.

    x_j = scale * (q . k_j);  out = sum_j exp(x_j - max x) v_j / sum_j exp(x_j - max x).
    ``scale`` is taken as the fp32 number the kernels receive, widened to fp64.
    An empty context gives a zero vector (reading adopted; the pages are silent).
    """
    q_head = np.asarray(q_head, dtype=np.float64)
    if k_rows.shape[0] == 0:
        return np.zeros(q_head.shape[0], dtype=np.float64)
    x = float(np.float32(scale)) * (k_rows @ q_head)
    w = np.exp(x - x.max())
    return (w @ v_rows) / w.sum()


def decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale):
    """Paged decode attention for a batch.

    q: [S][Hq][d]; k_cache, v_cache: [num_blocks][Hkv][B][d];
    block_tables: [S][max_blocks]; context_lens: [S].
    Returns out: [S][Hq][d] in fp64.
    """
    num_seqs, num_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[1]
    group = num_heads // num_kv_heads
    out = np.zeros((num_seqs, num_heads, head_dim), dtype=np.float64)
    for s in range(num_seqs):
        ctx = int(context_lens[s])
        for kvh in range(num_kv_heads):
            k_rows = gather_kv(k_cache, block_tables[s], ctx, kvh)
            v_rows = gather_kv(v_cache, block_tables[s], ctx, kvh)
            for h in range(kvh * group, (kvh + 1) * group):
                out[s, h] = decode_attention_one(q[s, h], k_rows, v_rows, scale)
    return out


def reshape_and_cache(key, value, k_cache, v_cache, slot_mapping):
    """Write each new token's K/V into its slot; returns new pool arrays.

    key, value: [T][Hkv][d]; slot_mapping: [T].  Token t goes to physical block
    slot // B at offset slot % B, for every kv head; slot < 0 writes nothing.
    Works on any dtype (bf16 pools travel as their raw 16-bit patterns), so the
    copy is bit-exact by construction.
    """
    k_out = k_cache.copy()
    v_out = v_cache.copy()
    block_size = k_cache.shape[2]
    for t in range(len(slot_mapping)):
        slot = int(slot_mapping[t])
        if slot < 0:
            continue
        block, offset = slot // block_size, slot % block_size
        for h in range(k_cache.shape[1]):
            k_out[block, h, offset, :] = key[t, h, :]
            v_out[block, h, offset, :] = value[t, h, :]
    return k_out, v_out


def copy_blocks(k_cache, v_cache, src_dst_pairs):
    """Copy-on-write block copies; returns new pool arrays.

    For every (src, dst) pair the whole physical block ``src`` (all kv heads,
    all B slots) is copied over block ``dst``, in both pools.  Sources are read
    from the pools as they were before any copy of this call.
    """
    k_out = k_cache.copy()
    v_out = v_cache.copy()
    for src, dst in src_dst_pairs:
        k_out[int(dst)] = k_cache[int(src)]
        v_out[int(dst)] = v_cache[int(src)]
    return k_out, v_out


def prefill_attention(q, k_cache, v_cache, block_tables, context_lens, query_start, scale):
    """Causal attention of a chunk of new tokens against the paged context.

    Sequence s holds context_lens[s] tokens; its last n_s = query_start[s+1] -
    query_start[s] tokens are the new ones, whose queries are rows
    query_start[s] .. query_start[s+1]-1 of q ([T][Hq][d]).  New token i of s sits
    at position pos = context_lens[s] - n_s + i and attends to the tokens at
    positions 0 .. pos of its own sequence (the prefill step of the
    "PagedAttention blog", section 3(3), over K/V read through the block table).
    Returns out [T][Hq][d] in fp64.
    """
    T, num_heads, head_dim = q.shape
    num_kv_heads = k_cache.shape[1]
    group = num_heads // num_kv_heads
    out = np.zeros((T, num_heads, head_dim), dtype=np.float64)
    for s in range(len(context_lens)):
        ctx = int(context_lens[s])
        first, last = int(query_start[s]), int(query_start[s + 1])
        n_new = last - first
        for kvh in range(num_kv_heads):
            k_rows = gather_kv(k_cache, block_tables[s], ctx, kvh)
            v_rows = gather_kv(v_cache, block_tables[s], ctx, kvh)
            for i in range(n_new):
                pos = ctx - n_new + i
                for h in range(kvh * group, (kvh + 1) * group):
                    out[first + i, h] = decode_attention_one(q[first + i, h], k_rows[: pos + 1],
                                                             v_rows[: pos + 1], scale)
    return out
