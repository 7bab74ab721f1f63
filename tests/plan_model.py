"""A plain Python model of the decode plan's work list.

The plan kernel turns context lengths and block tables into the list of work
items the attend kernel runs ("PagedAttention blog", section 4: parallel
samples map their logical blocks to the same physical blocks, so one read of a
shared block can serve all of them).  This model writes its rules out one
sequence at a time: whole partitions in sequence order, consecutive sequences
that share a partition's blocks packed (up to 8 x 3 / g of them, runs counted
from the start of each sharing chain and cut at the plan's chunk ends), shared
items of more than 8 columns split into 3 stream items while the workspace
holds split slots, then one item per ragged tail, longest length class first.
Item: (code, context, split slot or -1) with code = ((s * max_parts + p) << 7)
| (stream << 5) | (count - 1).
"""

import numpy as np

W_STREAMS = 3          # warps of the bf16 attend kernel: streams and column groups of a unit
SPLIT_CAP_MAX = 256    # split shared units the workspace holds
TAIL_CLASSES = 4
PLAN_THREADS = 1024


def model_plan(ctx, tables, P, B, Hq, Hkv, max_parts):
    """The work list of a bf16 decode batch, written from the rules above."""
    S = len(ctx)
    g = Hq // Hkv
    pack = 8 * W_STREAMS // g if g <= 8 else 1
    split_cap = min(SPLIT_CAP_MAX, (S // 2) * max_parts * Hq)
    split_items = split_cap // Hkv if pack > 1 else 0
    chunk = PLAN_THREADS if S >= PLAN_THREADS else (128 if S <= 128 else -(-S // 32) * 32)

    def code(s, p, count, stream=0):
        return ((s * max_parts + p) << 7) | (stream << 5) | (count - 1)

    # leading whole partitions each sequence shares with the next one
    lead = [0] * S
    for s in range(S - 1):
        if pack <= 1:
            continue
        kmax = min(ctx[s], ctx[s + 1]) // P
        k = 0
        while k < kmax and np.array_equal(tables[s, k * (P // B):(k + 1) * (P // B)],
                                          tables[s + 1, k * (P // B):(k + 1) * (P // B)]):
            k += 1
        lead[s] = k

    full, tails = [], [[] for _ in range(TAIL_CLASSES)]
    split_id = 0
    for start in range(0, S, chunk):
        end_chunk = min(start + chunk, S)
        chain = start
        for s in range(start, end_chunk):
            if s > start and lead[s - 1] == 0:
                chain = s
            c0 = chain + ((s - chain) // pack) * pack if pack > 1 else s
            end = min(c0 + pack, end_chunk)
            nfull = ctx[s] // P
            own_from = 0
            if pack > 1 and s == c0:
                kshared = min(nfull, lead[s]) if s + 1 < end else 0
                for k in range(kshared):
                    cnt = 2
                    while c0 + cnt < end and lead[c0 + cnt - 1] > k:
                        cnt += 1
                    if cnt * g > 8 and split_id < split_items:
                        full += [(code(s, k, cnt, st), ctx[s], split_id * Hkv) for st in range(W_STREAMS)]
                        split_id += 1
                        continue
                    if cnt * g > 8:
                        split_id += 1
                    full.append((code(s, k, cnt), ctx[s], -1))
                own_from = kshared
            elif pack > 1:
                own_from = nfull
                for t in range(c0, s):
                    own_from = min(own_from, lead[t])
            full += [(code(s, k, 1), ctx[s], -1) for k in range(own_from, nfull)]
            if ctx[s] % P != 0 or ctx[s] == 0:
                tails[((ctx[s] % P) * TAIL_CLASSES) // P].append((code(s, ctx[s] // P, 1), ctx[s], -1))
    items = full
    for b in reversed(range(TAIL_CLASSES)):
        items = items + tails[b]
    return items
