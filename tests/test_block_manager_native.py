"""The library's host block manager (pa_bm_*, C++) on CPU: lockstep with the
Python manager, the worked example of the "PagedAttention blog", and the
prefix-caching behaviour of "Month 2 · PagedAttention" section 04."""

import json
import os

import numpy as np
import pytest

from paged_kv_cache_382_b200.blocks import BlockManager, BlockPool

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example_parallel_sampling.json")


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


def test_lockstep_with_python_manager(pa):
    rng = np.random.default_rng(3)
    for trial in range(20):
        NB, B = int(rng.integers(8, 64)), int(rng.choice([1, 4, 16]))
        order = rng.permutation(NB)
        py = BlockManager(BlockPool(NB, order), B)
        nat = pa.NativeBlockManager(NB, B, order)
        live = {}
        next_id = 0
        for step in range(200):
            op = rng.integers(0, 10)
            if op < 2 or not live:                      # new sequence
                live[next_id] = py.new_sequence()
                nat.add(next_id)
                next_id += 1
            elif op < 3:                                # fork
                parent = int(rng.choice(list(live)))
                live[next_id] = py.fork(live[parent])
                nat.fork(parent, next_id)
                next_id += 1
            elif op < 4:                                # free
                sid = int(rng.choice(list(live)))
                py.free(live.pop(sid))
                nat.free(sid)
            else:                                       # append
                sid = int(rng.choice(list(live)))
                n = int(rng.integers(1, 3 * B + 2))
                try:
                    slots, copies = py.append_tokens(live[sid], n)
                    ok = True
                except RuntimeError:
                    ok = False
                if not ok:
                    break                               # pool exhausted: end this trial
                s2, c2, cached = nat.append(sid, n)
                assert list(s2) == slots and c2 == copies and cached == 0
            for sid, sq in live.items():
                assert nat.block_table(sid) == sq.block_table
                assert nat.num_tokens(sid) == sq.num_tokens
            assert nat.num_free == py.pool.num_free
            assert all(nat.ref_count(b) == py.pool.ref_cnt[b] for b in range(NB))


def test_worked_example(pa):
    gold = json.load(open(GOLDEN))
    m = pa.NativeBlockManager(8, 4, [7, 1, 3, 0, 2, 4, 5, 6])
    m.add(1)
    slots, copies, _ = m.append(1, 7)
    assert m.block_table(1) == gold["prefill"]["block_table"] and copies == []
    m.fork(1, 2)
    ps = gold["parallel_sampling"]
    assert all(m.ref_count(b) == ps["ref_count_shared"] for b in ps["shared_block_table"])
    _, c1, _ = m.append(1, 1)
    _, c2, _ = m.append(2, 1)
    assert c1 == [(1, ps["A1_new_physical_block"])] and c2 == []
    assert m.block_table(1) == ps["A1_block_table_after"] and m.block_table(2) == ps["A2_block_table_after"]
    for blk, ref in ps["ref_count_after"].items():
        assert m.ref_count(int(blk)) == ref


def test_prefix_cache_hit_skips_the_shared_block(pa):
    """Two requests with the same 16-token system prompt and different user
    tokens (5 and 6): the second references the first's block and has nothing
    to write for those 16 tokens."""
    rng = np.random.default_rng(5)
    system = rng.integers(0, 32000, size=16)
    r1 = np.concatenate([system, rng.integers(0, 32000, size=5)])
    r2 = np.concatenate([system, rng.integers(0, 32000, size=6)])
    m = pa.NativeBlockManager(32, 16, prefix_cache=True)
    m.add(1)
    s1, _, cached1 = m.append(1, r1)
    assert cached1 == 0 and np.all(s1 >= 0)
    m.add(2)
    s2, _, cached2 = m.append(2, r2)
    assert cached2 == 16 and np.all(s2[:16] == -1) and np.all(s2[16:] >= 0)
    assert m.block_table(2)[0] == m.block_table(1)[0]
    assert m.ref_count(m.block_table(1)[0]) == 2
    assert m.block_table(2)[1] != m.block_table(1)[1]


def test_prefix_keys_are_chained(pa):
    """The same 16 tokens after a different first block are a different key."""
    rng = np.random.default_rng(6)
    a, b = rng.integers(0, 32000, size=16), rng.integers(0, 32000, size=16)
    m = pa.NativeBlockManager(32, 16, prefix_cache=True)
    m.add(1)
    m.append(1, np.concatenate([a, b]))
    m.add(2)
    _, _, cached = m.append(2, np.concatenate([b, a]))
    assert cached == 0
    m.add(3)
    _, _, cached = m.append(3, np.concatenate([a, b, a]))
    assert cached == 32


def test_cached_block_survives_free_until_reused(pa):
    rng = np.random.default_rng(7)
    system = rng.integers(0, 32000, size=16)
    m = pa.NativeBlockManager(4, 16, prefix_cache=True)
    m.add(1)
    m.append(1, np.concatenate([system, [1, 2, 3]]))
    blk = m.block_table(1)[0]
    m.free(1)
    assert m.ref_count(blk) == 0 and m.num_free == 4
    m.add(2)                                      # still cached while free
    _, _, cached = m.append(2, np.concatenate([system, [9]]))
    assert cached == 16 and m.block_table(2)[0] == blk
    m.free(2)
    m.add(3)                                      # four fresh blocks: the cached one is reused and evicted
    m.append(3, rng.integers(0, 32000, size=64))
    m.free(3)
    m.add(4)
    _, _, cached = m.append(4, np.concatenate([system, [9]]))
    assert cached == 0


def test_errors(pa):
    m = pa.NativeBlockManager(2, 4)
    m.add(1)
    with pytest.raises(pa.PagedAttentionError):
        m.add(1)
    with pytest.raises(pa.PagedAttentionError):
        m.fork(7, 8)
    with pytest.raises(pa.PagedAttentionError):
        m.append(1, 9)                            # needs 3 blocks of 4 slots, the pool has 2
    assert pa.lib.pa_bm_create(0, 4, None, 0) is None
    bad = np.array([0, 0], dtype=np.int32)
    assert pa.lib.pa_bm_create(2, 4, bad.ctypes.data, 0) is None


@pytest.mark.parametrize("prefix_cache", [False, True], ids=["plain", "prefix_cache"])
def test_append_batch_equals_one_call_per_sequence(pa, prefix_cache):
    """pa_bm_append_batch gives the same slots, copy-on-write pairs, cached counts
    and resulting tables as one pa_bm_append per sequence, in order."""
    rng = np.random.default_rng(11)
    NB, B = 400, 16
    a = pa.NativeBlockManager(NB, B, prefix_cache=prefix_cache)
    b = pa.NativeBlockManager(NB, B, prefix_cache=prefix_cache)
    system = rng.integers(1, 1000, size=40).tolist()
    seqs = []
    for sid in range(6):                                   # prompts, some with a shared system prompt
        toks = (system if sid % 2 == 0 else []) + rng.integers(1, 1000, size=int(rng.integers(1, 30))).tolist()
        for m in (a, b):
            m.add(sid)
        ra, rb = a.append(sid, toks if prefix_cache else len(toks)), b.append_batch([sid], [toks if prefix_cache
                                                                                       else len(toks)])
        assert list(ra[0]) == list(rb[0]) and ra[1] == rb[1] and ra[2] == rb[2]
        seqs.append(sid)
    for child, parent in [(6, 0), (7, 0), (8, 3)]:       # parallel samples
        a.fork(parent, child)
        b.fork(parent, child)
        seqs.append(child)
    for step in range(12):                                 # decode steps: 1-3 tokens per sequence
        batch = [rng.integers(1, 1000, size=int(rng.integers(1, 4))).tolist() for _ in seqs]
        want_slots, want_copies, want_cached = [], [], 0
        for sid, toks in zip(seqs, batch):
            s, c, k = a.append(sid, toks if prefix_cache else len(toks))
            want_slots += list(s)
            want_copies += c
            want_cached += k
        if step % 2 == 0:
            got_slots, got_copies, got_cached = b.append_batch(seqs, batch if prefix_cache
                                                               else [len(t) for t in batch])
        else:                                              # flat arrays, as a serving loop holds them
            flat = np.concatenate([np.asarray(t, dtype=np.int32) for t in batch]) if prefix_cache else None
            got_slots, got_copies, got_cached = b.append_batch(np.asarray(seqs), flat,
                                                               counts=[len(t) for t in batch])
        assert list(got_slots) == want_slots and got_copies == want_copies and got_cached == want_cached
    for sid in seqs:
        assert a.block_table(sid) == b.block_table(sid)
    assert a.num_free == b.num_free


def test_append_batch_validation(pa):
    m = pa.NativeBlockManager(8, 4)
    m.add(0)
    with pytest.raises(Exception):
        m.append_batch([0, 5], [1, 1])                     # unknown id: nothing changes
    assert m.num_tokens(0) == 0 and m.num_free == 8
    with pytest.raises(Exception):
        m.append_batch([0], [-1])                          # negative count
    with pytest.raises(ValueError):
        pa.NativeBlockManager(8, 4, prefix_cache=True).append_batch([0], np.zeros(3, np.int32), counts=[2])
    slots, copies, cached = m.append_batch([], [])
    assert len(slots) == 0 and copies == [] and cached == 0
    slots, copies, _ = m.append_batch([0, 0], [3, 2])      # a sequence twice: appended in order
    assert list(slots) == [0, 1, 2, 3, 4]                  # blocks 0 then 1 (default free order)
    assert m.num_tokens(0) == 5
