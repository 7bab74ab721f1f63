"""Pins for the fp64 oracle and the host block manager (CPU only).

Each check ties the oracle to something other than itself: the worked example
printed on the "PagedAttention blog" (sections 3(3) and 4), torch's own
scaled_dot_product_attention on contiguous K/V (the pages' statement that the
paged kernel is ordinary attention over logically contiguous tokens), closed
forms of special cases, a pure-Python brute force, and invariants the pages
fix (physical placement is transparent, shared blocks give the same result,
copy-on-write isolates sharers).  ``test_mutants_are_caught`` plants plausible
mistakes in copies of the oracle and checks that some pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from paged_kv_cache_382_b200.blocks import BlockManager, BlockPool, block_table_array

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_parallel_sampling.json")


def load_golden():
    with open(GOLDEN) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# helpers that build paged inputs from contiguous ones without slot arithmetic
# --------------------------------------------------------------------------

def paged_from_contiguous(k_seqs, v_seqs, block_size, rng, spare_blocks=3, pad_value=np.nan):
    """Lay each sequence's contiguous K/V [Hkv][ctx][d] into whole blocks, then move
    every block to a random physical id.  Returns pools and block tables."""
    Hkv, d = k_seqs[0].shape[0], k_seqs[0].shape[2]
    blocks_k, blocks_v, owners = [], [], []
    for s, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        ctx = k.shape[1]
        nb = -(-ctx // block_size)
        padded_k = np.full((Hkv, nb * block_size, d), pad_value)
        padded_v = np.full((Hkv, nb * block_size, d), pad_value)
        padded_k[:, :ctx] = k
        padded_v[:, :ctx] = v
        for i in range(nb):
            blocks_k.append(padded_k[:, i * block_size:(i + 1) * block_size])
            blocks_v.append(padded_v[:, i * block_size:(i + 1) * block_size])
            owners.append(s)
    n_used = len(blocks_k)
    num_blocks = n_used + spare_blocks
    perm = rng.permutation(num_blocks)[:n_used]
    k_cache = np.full((num_blocks, Hkv, block_size, d), pad_value)
    v_cache = np.full((num_blocks, Hkv, block_size, d), pad_value)
    max_blocks = max(1, max(-(-k.shape[1] // block_size) for k in k_seqs)) + 2
    tables = np.full((len(k_seqs), max_blocks), -1, dtype=np.int64)
    fill = [0] * len(k_seqs)
    for j in range(n_used):
        k_cache[perm[j]] = blocks_k[j]
        v_cache[perm[j]] = blocks_v[j]
        s = owners[j]
        tables[s, fill[s]] = perm[j]
        fill[s] += 1
    return k_cache, v_cache, tables


def sdpa_contiguous(q, k_seqs, v_seqs, scale):
    """torch's scaled_dot_product_attention in fp64 on contiguous K/V, per sequence."""
    outs = []
    Hq = q.shape[1]
    for s, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        Hkv = k.shape[0]
        if k.shape[1] == 0:
            outs.append(np.zeros((Hq, q.shape[2])))
            continue
        qt = torch.from_numpy(q[s][:, None, :]).double()[None]          # [1][Hq][1][d]
        kt = torch.from_numpy(k).double()[None]                          # [1][Hkv][ctx][d]
        vt = torch.from_numpy(v).double()[None]
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, scale=float(np.float32(scale)), enable_gqa=(Hq != Hkv))
        outs.append(o[0, :, 0, :].numpy())
    return np.stack(outs)


def random_problem(rng, ctx_lens, Hq, Hkv, d, block_size, scale=None):
    k_seqs = [rng.standard_normal((Hkv, c, d)) for c in ctx_lens]
    v_seqs = [rng.standard_normal((Hkv, c, d)) for c in ctx_lens]
    q = rng.standard_normal((len(ctx_lens), Hq, d))
    k_cache, v_cache, tables = paged_from_contiguous(k_seqs, v_seqs, block_size, rng)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return dict(q=q, k_seqs=k_seqs, v_seqs=v_seqs, k_cache=k_cache, v_cache=v_cache,
                tables=tables, ctx=np.array(ctx_lens), scale=scale)


def brute_force(q, k_cache, v_cache, tables, ctx_lens, scale):
    """Pure-Python loops: find each token's row by walking the table, then the
    textbook softmax-weighted sum with the running max subtracted."""
    S, Hq, d = q.shape
    Hkv, B = k_cache.shape[1], k_cache.shape[2]
    g = Hq // Hkv
    out = np.zeros((S, Hq, d))
    sc = float(np.float32(scale))
    for s in range(S):
        for h in range(Hq):
            kvh = h // g
            logits = []
            for j in range(int(ctx_lens[s])):
                row = k_cache[int(tables[s][j // B]), kvh, j % B]
                logits.append(sc * sum(float(q[s, h, e]) * float(row[e]) for e in range(d)))
            if not logits:
                continue
            top = max(logits)
            w = [math.exp(x - top) for x in logits]
            total = math.fsum(w)
            for e in range(d):
                acc = math.fsum(w[j] * float(v_cache[int(tables[s][j // B]), kvh, j % B, e])
                                for j in range(len(w)))
                out[s, h, e] = acc / total
    return out


# --------------------------------------------------------------------------
# pin checks, written as functions so the mutant test can rerun them
# --------------------------------------------------------------------------

def pin_sdpa(decode):
    rng = np.random.default_rng(1)
    ok = True
    for ctx, Hq, Hkv, d, B in [([7, 16, 33, 100], 4, 4, 64, 16), ([7, 16, 33, 100], 4, 4, 64, 4),
                               ([1, 5, 64, 29], 8, 2, 32, 8), ([3, 40], 6, 3, 16, 32)]:
        p = random_problem(rng, ctx, Hq, Hkv, d, B)
        got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
        ref = sdpa_contiguous(p["q"], p["k_seqs"], p["v_seqs"], p["scale"])
        ok &= bool(np.all(np.isfinite(got))) and float(np.abs(got - ref).max()) <= 1e-12
    return ok


def pin_brute_force(decode):
    rng = np.random.default_rng(2)
    p = random_problem(rng, [1, 2, 5, 9], 4, 2, 8, 4)
    got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    ref = brute_force(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    return bool(np.all(np.isfinite(got))) and float(np.abs(got - ref).max()) <= 1e-12


def pin_special_cases(decode):
    rng = np.random.default_rng(3)
    ok = True
    # ctx = 1: the only weight is exp(0)/1, so out is the single value row exactly
    p = random_problem(rng, [1, 1], 2, 2, 16, 4)
    got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    for s in range(2):
        for h in range(2):
            ok &= bool(np.array_equal(got[s, h], p["v_seqs"][s][h, 0]))
    # q = 0: all logits equal, out is the plain mean of the value rows
    p = random_problem(rng, [13, 4], 2, 1, 16, 4)
    p["q"][:] = 0.0
    got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    for s in range(2):
        mean = p["v_seqs"][s][0].mean(axis=0)
        ok &= float(np.abs(got[s] - mean[None]).max()) <= 1e-14
    # ctx = 0: zeros (reading adopted for an empty context)
    p = random_problem(rng, [0, 3], 2, 2, 8, 4)
    got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    ok &= bool(np.all(got[0] == 0.0))
    # large logits: scale x 100 must stay finite and match scipy's softmax
    p = random_problem(rng, [37, 5], 4, 2, 16, 8, scale=100.0 / 4.0)
    got = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    ok &= bool(np.all(np.isfinite(got)))
    for s in range(2):
        for h in range(4):
            k = p["k_seqs"][s][h // 2]
            v = p["v_seqs"][s][h // 2]
            w = scipy.special.softmax(float(np.float32(p["scale"])) * (k @ p["q"][s, h]))
            ok &= float(np.abs(got[s, h] - w @ v).max()) <= 1e-12
    return ok


def pin_permutation(decode):
    rng = np.random.default_rng(4)
    p = random_problem(rng, [9, 30, 17], 4, 2, 16, 4)
    base = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    NB = p["k_cache"].shape[0]
    perm = rng.permutation(NB)
    k2 = np.empty_like(p["k_cache"])
    v2 = np.empty_like(p["v_cache"])
    k2[perm] = p["k_cache"]
    v2[perm] = p["v_cache"]
    t2 = np.where(p["tables"] >= 0, perm[np.maximum(p["tables"], 0)], -1)
    moved = decode(p["q"], k2, v2, t2, p["ctx"], p["scale"])
    return bool(np.array_equal(base, moved))


def pin_shared_blocks(decode):
    rng = np.random.default_rng(5)
    p = random_problem(rng, [21, 21], 2, 2, 16, 4)
    q = p["q"].copy()
    q[1] = q[0]
    tables = p["tables"].copy()
    shared = decode(q, p["k_cache"], p["v_cache"], np.stack([tables[0], tables[0]]), p["ctx"], p["scale"])
    ok = bool(np.array_equal(shared[0], shared[1]))
    # same contents in different blocks: copy seq 0's blocks over seq 1's
    k2, v2 = p["k_cache"].copy(), p["v_cache"].copy()
    for i in range(-(-21 // 4)):
        k2[tables[1, i]] = k2[tables[0, i]]
        v2[tables[1, i]] = v2[tables[0, i]]
    dup = decode(q, k2, v2, tables, p["ctx"], p["scale"])
    ok &= bool(np.array_equal(dup[0], dup[1]))
    return ok


def pin_masking(decode):
    rng = np.random.default_rng(6)
    p = random_problem(rng, [6, 13, 4], 4, 4, 16, 4)   # reservation slots are NaN already
    base = decode(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    # every free block NaN too, every table entry past the end -1
    used = set(int(b) for b in p["tables"].ravel() if b >= 0)
    k2, v2 = p["k_cache"].copy(), p["v_cache"].copy()
    for b in range(k2.shape[0]):
        if b not in used:
            k2[b] = np.nan
            v2[b] = np.nan
    again = decode(p["q"], k2, v2, p["tables"], p["ctx"], p["scale"])
    return bool(np.all(np.isfinite(base))) and bool(np.array_equal(base, again))


DECODE_PINS = [pin_sdpa, pin_brute_force, pin_special_cases, pin_permutation, pin_shared_blocks, pin_masking]


@pytest.mark.parametrize("pin", DECODE_PINS, ids=lambda f: f.__name__)
def test_decode_pin(pin):
    assert pin(oracle.decode_attention)


# --------------------------------------------------------------------------
# worked example of the "PagedAttention blog" (sections 3(3) and 4)
# --------------------------------------------------------------------------

def example_manager():
    pool = BlockPool(8, free_order=[7, 1, 3, 0, 2, 4, 5, 6])
    return BlockManager(pool, block_size=4)


def test_worked_example_prefill_and_decode():
    gold = load_golden()
    mgr = example_manager()
    seq = mgr.new_sequence()
    slots, copies = mgr.append_tokens(seq, len(gold["prompt"]))
    assert len(seq.block_table) == gold["prefill"]["num_logical_blocks"]
    assert seq.block_table == gold["prefill"]["block_table"]
    assert seq.filled(4) == gold["prefill"]["filled"]
    assert copies == []
    mgr.append_tokens(seq, 1)                     # "fathers"
    assert seq.filled(4) == gold["first_decode"]["filled_after"]
    assert seq.block_table == gold["prefill"]["block_table"]
    mgr.append_tokens(seq, 1)                     # the next token opens logical block 2
    assert len(seq.block_table) == gold["first_decode"]["next_token_opens_logical_block"] + 1


def test_worked_example_parallel_sampling():
    gold = load_golden()["parallel_sampling"]
    mgr = example_manager()
    a1 = mgr.new_sequence()
    mgr.append_tokens(a1, 7)
    a2 = mgr.fork(a1)
    assert a1.block_table == a2.block_table == gold["shared_block_table"]
    assert all(mgr.pool.ref_cnt[b] == gold["ref_count_shared"] for b in gold["shared_block_table"])
    _, copies_a1 = mgr.append_tokens(a1, 1)       # A1 writes "fathers" into shared block 1
    assert copies_a1 == [(1, gold["A1_new_physical_block"])]
    _, copies_a2 = mgr.append_tokens(a2, 1)       # A2 writes "mothers": last sharer, in place
    assert copies_a2 == []
    assert a1.block_table == gold["A1_block_table_after"]
    assert a2.block_table == gold["A2_block_table_after"]
    for blk, ref in gold["ref_count_after"].items():
        assert mgr.pool.ref_cnt[int(blk)] == ref


def test_scatter_places_prompt_in_example_blocks():
    """Prefill of the example: tokens 0-3 land in physical block 7, tokens 4-6 in
    block 1, and block 1's fourth slot (the reservation) is left alone."""
    mgr = example_manager()
    seq = mgr.new_sequence()
    slots, _ = mgr.append_tokens(seq, 7)
    rng = np.random.default_rng(7)
    key = rng.standard_normal((7, 2, 8))
    value = rng.standard_normal((7, 2, 8))
    sentinel = -12345.0
    k_cache = np.full((8, 2, 4, 8), sentinel)
    v_cache = np.full((8, 2, 4, 8), sentinel)
    k2, v2 = oracle.reshape_and_cache(key, value, k_cache, v_cache, np.array(slots))
    for t in range(4):
        assert np.array_equal(k2[7, :, t], key[t]) and np.array_equal(v2[7, :, t], value[t])
    for t in range(4, 7):
        assert np.array_equal(k2[1, :, t - 4], key[t]) and np.array_equal(v2[1, :, t - 4], value[t])
    assert np.all(k2[1, :, 3] == sentinel) and np.all(v2[1, :, 3] == sentinel)
    others = [b for b in range(8) if b not in (7, 1)]
    assert np.all(k2[others] == sentinel) and np.all(v2[others] == sentinel)


def pin_scatter_roundtrip(scatter):
    """Scatter every token through the manager's slots, gather through the block
    table: the contiguous K/V come back exactly; nothing else is touched; a
    negative slot writes nothing."""
    rng = np.random.default_rng(8)
    ok = True
    for B, lens in [(4, [7, 1, 12]), (16, [33, 16]), (8, [0, 9, 17])]:
        pool = BlockPool(24, free_order=rng.permutation(24))
        mgr = BlockManager(pool, B)
        seqs, slots = [], []
        for c in lens:
            sq = mgr.new_sequence()
            sl, _ = mgr.append_tokens(sq, c)
            seqs.append(sq)
            slots.extend(sl)
        T = len(slots)
        key = rng.standard_normal((T + 1, 3, 4))
        value = rng.standard_normal((T + 1, 3, 4))
        slot_arr = np.array(slots + [-1])
        kc = np.full((24, 3, B, 4), 7.5)
        vc = np.full((24, 3, B, 4), 7.5)
        k2, v2 = scatter(key, value, kc, vc, slot_arr)
        tables = block_table_array(seqs)
        off = 0
        for sq, c in zip(seqs, lens):
            for h in range(3):
                ok &= bool(np.array_equal(oracle.gather_kv(k2, sq.block_table, c, h), key[off:off + c, h]))
                ok &= bool(np.array_equal(oracle.gather_kv(v2, sq.block_table, c, h), value[off:off + c, h]))
            off += c
        written = int(np.sum(k2 != 7.5))
        ok &= written == T * 3 * 4
        ok &= int(np.sum(v2 != 7.5)) == T * 3 * 4
        del tables
    return ok


def pin_copy_on_write(copy):
    """Section 4 example at the pool level: after the copy of block 1 into block 3,
    block 3 equals block 1, block 1 is unchanged, every other block is untouched;
    sources are read before any copy of the same call lands."""
    rng = np.random.default_rng(9)
    kc = rng.standard_normal((8, 2, 4, 8))
    vc = rng.standard_normal((8, 2, 4, 8))
    k2, v2 = copy(kc, vc, [(1, 3)])
    ok = bool(np.array_equal(k2[3], kc[1]) and np.array_equal(v2[3], vc[1]))
    ok &= bool(np.array_equal(k2[1], kc[1]) and np.array_equal(v2[1], vc[1]))
    rest = [b for b in range(8) if b != 3]
    ok &= bool(np.array_equal(k2[rest], kc[rest]) and np.array_equal(v2[rest], vc[rest]))
    k3, v3 = copy(kc, vc, [(0, 5), (2, 6)])
    ok &= bool(np.array_equal(k3[5], kc[0]) and np.array_equal(k3[6], kc[2]))
    ok &= bool(np.array_equal(v3[5], vc[0]) and np.array_equal(v3[6], vc[2]))
    return ok


def test_scatter_roundtrip():
    assert pin_scatter_roundtrip(oracle.reshape_and_cache)


def test_copy_on_write_blocks():
    assert pin_copy_on_write(oracle.copy_blocks)


def test_copy_on_write_isolates_sharers():
    """A1 and A2 share [7, 1]; A1 copies block 1 to 3 and writes 'fathers' at
    slot 3*4+3, A2 writes 'mothers' at slot 1*4+3.  A2's output is identical
    before and after A1's write, and each sample's output is ordinary attention
    over its own eight tokens."""
    rng = np.random.default_rng(10)
    Hkv, d = 2, 16
    mgr = example_manager()
    a1 = mgr.new_sequence()
    prompt_slots, _ = mgr.append_tokens(a1, 7)
    a2 = mgr.fork(a1)
    prompt_k = rng.standard_normal((7, Hkv, d))
    prompt_v = rng.standard_normal((7, Hkv, d))
    kc = np.full((8, Hkv, 4, d), np.nan)
    vc = np.full((8, Hkv, 4, d), np.nan)
    kc, vc = oracle.reshape_and_cache(prompt_k, prompt_v, kc, vc, np.array(prompt_slots))
    s1, c1 = mgr.append_tokens(a1, 1)
    s2, c2 = mgr.append_tokens(a2, 1)
    q = rng.standard_normal((2, Hkv, d))
    scale = 0.25
    # A2's view with its own token written but before A1's copy and write
    tok_k = rng.standard_normal((2, Hkv, d))
    tok_v = rng.standard_normal((2, Hkv, d))
    kb, vb = oracle.reshape_and_cache(tok_k[1:], tok_v[1:], kc, vc, np.array(s2))
    before = oracle.decode_attention(q[1:], kb, vb, np.array([a2.block_table]), np.array([8]), scale)
    kc2, vc2 = oracle.copy_blocks(kc, vc, c1 + c2)
    assert np.array_equal(kc2[3, :, :3], kc2[1, :, :3]) and np.array_equal(vc2[3, :, :3], vc2[1, :, :3])
    kc3, vc3 = oracle.reshape_and_cache(tok_k, tok_v, kc2, vc2, np.array(s1 + s2))
    assert s1 == [15] and s2 == [7]
    after = oracle.decode_attention(q, kc3, vc3, np.array([a1.block_table, a2.block_table]),
                                    np.array([8, 8]), scale)
    assert np.array_equal(after[1], before[0])
    for i in range(2):
        k_seq = np.concatenate([prompt_k, tok_k[i:i + 1]]).transpose(1, 0, 2)
        v_seq = np.concatenate([prompt_v, tok_v[i:i + 1]]).transpose(1, 0, 2)
        ref = sdpa_contiguous(q[i:i + 1], [k_seq], [v_seq], scale)
        assert float(np.abs(after[i] - ref[0]).max()) <= 1e-12


# --------------------------------------------------------------------------
# planted mistakes: every mutant of the oracle must fail some pin
# --------------------------------------------------------------------------

def _mutant_decode(kind):
    def decode(q, k_cache, v_cache, block_tables, context_lens, scale):
        S, Hq, d = q.shape
        Hkv, B = k_cache.shape[1], k_cache.shape[2]
        g = Hq // Hkv
        out = np.zeros((S, Hq, d))
        for s in range(S):
            ctx = int(context_lens[s])
            n_used = ctx - 1 if kind == "drop_last_token" else ctx
            if kind == "keep_reservation":
                n_used = -(-ctx // B) * B
            for h in range(Hq):
                kvh = h % Hkv if kind == "gqa_modulo" else h // g
                table = np.arange(block_tables.shape[1]) if kind == "ignore_table" else block_tables[s]
                k_rows = oracle.gather_kv(k_cache, table, n_used, kvh) if n_used > 0 else np.zeros((0, d))
                v_rows = oracle.gather_kv(v_cache, table, n_used, kvh) if n_used > 0 else np.zeros((0, d))
                if kind == "keep_reservation" and n_used > 0:
                    pieces = [k_cache[int(table[i]), kvh] for i in range(n_used // B)]
                    k_rows = np.concatenate(pieces)
                    v_rows = np.concatenate([v_cache[int(table[i]), kvh] for i in range(n_used // B)])
                if kind == "values_are_keys":
                    v_rows = k_rows
                if k_rows.shape[0] == 0:
                    continue
                sc = 1.0 if kind == "no_scale" else float(np.float32(scale))
                x = sc * (k_rows @ q[s, h])
                if kind == "no_max_subtraction":
                    w = np.exp(x)
                else:
                    w = np.exp(x - x.max())
                o = w @ v_rows
                out[s, h] = o if kind == "no_normalisation" else o / w.sum()
        return out
    return decode


DECODE_MUTANTS = ["gqa_modulo", "no_scale", "drop_last_token", "keep_reservation", "ignore_table",
                  "values_are_keys", "no_max_subtraction", "no_normalisation"]


def _mutant_scatter(kind):
    def scatter(key, value, k_cache, v_cache, slot_mapping):
        k_out, v_out = k_cache.copy(), v_cache.copy()
        B = k_cache.shape[2]
        for t, slot in enumerate(slot_mapping):
            slot = int(slot)
            if slot < 0 and kind != "negative_slot_written":
                continue
            blk, off = (slot % B, slot // B) if kind == "swapped_divmod" else (slot // B, slot % B)
            if blk >= k_cache.shape[0]:
                continue
            k_out[blk, :, off] = key[t]
            v_out[blk, :, off] = key[t] if kind == "value_from_key" else value[t]
        return k_out, v_out
    return scatter


def _mutant_copy(kind):
    def copy(k_cache, v_cache, pairs):
        k_out, v_out = k_cache.copy(), v_cache.copy()
        for src, dst in pairs:
            if kind == "reversed":
                src, dst = dst, src
            k_out[dst] = k_cache[src]
            if kind != "keys_only":
                v_out[dst] = (k_out if kind == "values_from_keys" else v_cache)[src]
        return k_out, v_out
    return copy


@pytest.mark.parametrize("kind", DECODE_MUTANTS)
def test_decode_mutants_are_caught(kind):
    mutant = _mutant_decode(kind)
    failures = []
    for pin in DECODE_PINS:
        try:
            ok = pin(mutant)
        except Exception:
            ok = False
        if not ok:
            failures.append(pin.__name__)
    assert failures, f"no pin catches the mutant {kind}"


@pytest.mark.parametrize("kind", ["swapped_divmod", "negative_slot_written", "value_from_key"])
def test_scatter_mutants_are_caught(kind):
    try:
        ok = pin_scatter_roundtrip(_mutant_scatter(kind))
    except Exception:
        ok = False
    assert not ok


@pytest.mark.parametrize("kind", ["reversed", "keys_only", "values_from_keys"])
def test_copy_mutants_are_caught(kind):
    try:
        ok = pin_copy_on_write(_mutant_copy(kind))
    except Exception:
        ok = False
    assert not ok


# --------------------------------------------------------------------------
# prefill (a chunk of new tokens, causal) against the paged context
# --------------------------------------------------------------------------

def prefill_problem(rng, ctx_lens, new_lens, Hq, Hkv, d, B):
    p = random_problem(rng, ctx_lens, Hq, Hkv, d, B)
    qs = np.concatenate([[0], np.cumsum(new_lens)]).astype(np.int64)
    p["q"] = rng.standard_normal((int(qs[-1]), Hq, d))
    p["query_start"] = qs
    return p


def pin_prefill_sdpa(prefill):
    """torch SDPA in fp64 with an explicit mask: new token i of a sequence with
    ctx tokens sees positions <= ctx - n + i."""
    rng = np.random.default_rng(12)
    ok = True
    for ctx, new, Hq, Hkv, d, B in [([7, 33, 100], [3, 33, 1], 4, 4, 16, 4), ([50, 17], [20, 5], 8, 2, 32, 16)]:
        p = prefill_problem(rng, ctx, new, Hq, Hkv, d, B)
        got = prefill(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["query_start"], p["scale"])
        for s, (c, n) in enumerate(zip(ctx, new)):
            first = int(p["query_start"][s])
            qt = torch.from_numpy(p["q"][first:first + n].transpose(1, 0, 2).copy())[None]   # [1][Hq][n][d]
            kt = torch.from_numpy(p["k_seqs"][s])[None]
            vt = torch.from_numpy(p["v_seqs"][s])[None]
            pos = torch.arange(c - n, c)[:, None]
            mask = torch.arange(c)[None, :] <= pos                                            # [n][c]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qt, kt, vt, attn_mask=mask, scale=float(np.float32(p["scale"])), enable_gqa=(Hq != Hkv))
            ref = ref[0].numpy().transpose(1, 0, 2)
            ok &= float(np.abs(got[first:first + n] - ref).max()) <= 1e-12
    return ok


def pin_prefill_last_token_is_decode(prefill):
    """The last new token of every sequence sees the whole context: it equals decode."""
    rng = np.random.default_rng(13)
    p = prefill_problem(rng, [9, 40, 3], [4, 1, 3], 4, 2, 16, 8)
    got = prefill(p["q"], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["query_start"], p["scale"])
    last = p["query_start"][1:] - 1
    dec = oracle.decode_attention(p["q"][last], p["k_cache"], p["v_cache"], p["tables"], p["ctx"], p["scale"])
    return bool(np.array_equal(got[last], dec))


def test_prefill_pins():
    assert pin_prefill_sdpa(oracle.prefill_attention)
    assert pin_prefill_last_token_is_decode(oracle.prefill_attention)


def _mutant_prefill(kind):
    def prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale):
        T, Hq, d = q.shape
        Hkv = k_cache.shape[1]
        g = Hq // Hkv
        out = np.zeros((T, Hq, d))
        for s in range(len(context_lens)):
            ctx = int(context_lens[s])
            first, last = int(query_start[s]), int(query_start[s + 1])
            n = last - first
            for kvh in range(Hkv):
                K = oracle.gather_kv(k_cache, block_tables[s], ctx, kvh)
                V = oracle.gather_kv(v_cache, block_tables[s], ctx, kvh)
                for i in range(n):
                    pos = {"no_causal_mask": ctx - 1, "positions_from_zero": i,
                           "off_by_one": ctx - n + i - 1}.get(kind, ctx - n + i)
                    for h in range(kvh * g, (kvh + 1) * g):
                        out[first + i, h] = oracle.decode_attention_one(q[first + i, h], K[:pos + 1], V[:pos + 1],
                                                                        scale)
        return out
    return prefill


@pytest.mark.parametrize("kind", ["no_causal_mask", "positions_from_zero", "off_by_one"])
def test_prefill_mutants_are_caught(kind):
    assert not (pin_prefill_sdpa(_mutant_prefill(kind)) and pin_prefill_last_token_is_decode(_mutant_prefill(kind)))
