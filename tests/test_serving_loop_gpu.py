"""A small serving loop on the GPU, every step through the C ABI, checked
against plain attention over each sequence's contiguous K/V history.

The host block manager (``pa_bm_*``, prefix cache on) admits two requests that
share a 32-token system prompt: the second one finds the prompt's two full
blocks cached, so only its own tokens are written and prefilled (chunked
prefill on the tensor-core path).  The first request is then forked into two
parallel samples, and three decode steps run for all three sequences: the
manager's slots and copy-on-write pairs drive ``pa_copy_blocks``,
``pa_reshape_and_cache`` and ``pa_decode``.

The history of a sequence is the list of (K, V) of its tokens in order, built
on the host without any paging ("PagedAttention blog", section 3(3): attention
is computed as if the tokens were contiguous; the block table only says where
they are).  K/V of a token are a function of its position and id, so a cached
prefix holds exactly the values a recomputation would write.
"""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

HQ, HKV, D, B, NB = 16, 4, 128, 16, 64
TOL = 2e-3


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


def kv_of(pos: int, tok: int):
    """K, V [Hkv][d] of token id `tok` at position `pos`, bf16-representable."""
    rng = np.random.default_rng((pos * 1_000_003 + tok) & 0xFFFFFFFF)
    k = torch.from_numpy(rng.standard_normal((HKV, D))).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((HKV, D))).to(torch.bfloat16)
    return k, v


def reference(q_row: np.ndarray, hist, scale: float) -> np.ndarray:
    """q_row [Hq][d] against the contiguous history [(k, v), ...]."""
    k = np.stack([h[0].double().numpy() for h in hist])   # [T][Hkv][d]
    v = np.stack([h[1].double().numpy() for h in hist])
    g = HQ // HKV
    return np.stack([oracle.decode_attention_one(q_row[h], k[:, h // g], v[:, h // g], scale) for h in range(HQ)])


def test_prefix_cache_chunked_prefill_fork_and_decode(pa):
    dev = "cuda"
    scale = float(np.float32(1.0 / np.sqrt(D)))
    kc = torch.zeros(NB, HKV, B, D, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    bm = pa.NativeBlockManager(NB, B, prefix_cache=True)
    rng = np.random.default_rng(17)
    system = rng.integers(1, 30000, size=32).tolist()
    hist, ids = {}, {}

    def write(seq, toks, slots):
        """K/V of the seq's new tokens into the pool (cached tokens: slot -1, skipped)."""
        start = len(hist.get(seq, []))
        kv = [kv_of(start + i, t) for i, t in enumerate(toks)]
        hist.setdefault(seq, []).extend(kv)
        ids.setdefault(seq, []).extend(toks)
        key = torch.stack([x[0] for x in kv]).to(dev)
        val = torch.stack([x[1] for x in kv]).to(dev)
        pa.reshape_and_cache(key, val, kc, vc, torch.from_numpy(np.asarray(slots, dtype=np.int64)).to(dev),
                             dev_err=err)

    def tables(seqs):
        rows = [bm.block_table(s) for s in seqs]
        width = max(len(r) for r in rows)
        return np.array([r + [-1] * (width - len(r)) for r in rows], dtype=np.int32)

    # admission: request 0 (system prompt + 8 tokens) and request 1 (same prompt + 12)
    prompts = {0: system + rng.integers(1, 30000, size=8).tolist(),
               1: system + rng.integers(1, 30000, size=12).tolist()}
    new_counts = {}
    for s, toks in prompts.items():
        bm.add(s)
        slots, copies, cached = bm.append(s, toks)
        assert copies == []
        assert cached == (0 if s == 0 else 32)          # request 1 hits the cached prompt
        assert all(x == -1 for x in slots[:cached])
        write(s, toks, slots)
        new_counts[s] = len(toks) - cached

    # chunked prefill of the uncached tokens only (tensor-core path)
    assert pa.prefill_uses_tensor_cores(torch.bfloat16, HQ, HKV, D, B)
    seqs = [0, 1]
    T = sum(new_counts[s] for s in seqs)
    q = (torch.randn(T, HQ, D, generator=torch.Generator().manual_seed(3))).to(torch.bfloat16)
    qs = np.concatenate([[0], np.cumsum([new_counts[s] for s in seqs])]).astype(np.int32)
    ctx = np.array([len(hist[s]) for s in seqs], dtype=np.int32)
    out = torch.empty(T, HQ, D, dtype=torch.float32, device=dev)
    pa.prefill(out, q.to(dev), kc, vc, torch.from_numpy(tables(seqs)).to(dev), torch.from_numpy(ctx).to(dev),
               torch.from_numpy(qs).to(dev), scale, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    got = out.double().cpu().numpy()
    for j, s in enumerate(seqs):
        n = new_counts[s]
        for i in range(n):
            pos = len(hist[s]) - n + i
            ref = reference(q[qs[j] + i].double().numpy(), hist[s][: pos + 1], scale)
            assert np.abs(got[qs[j] + i] - ref).max() <= TOL, (s, i)

    # parallel sampling: request 0 forks into sequence 2; three decode steps
    bm.fork(0, 2)
    hist[2], ids[2] = list(hist[0]), list(ids[0])
    seqs = [0, 2, 1]
    total_copies = 0
    for step in range(3):
        new_tok = {s: int(rng.integers(1, 30000)) for s in seqs}
        slots, pairs = [], []
        for s in seqs:
            sl, cp, _ = bm.append(s, [new_tok[s]])
            slots.append(int(sl[0]))
            pairs += cp
        total_copies += len(pairs)
        if pairs:   # copy-on-write before the writes
            pa.copy_blocks(kc, vc, torch.tensor(pairs, dtype=torch.int64, device=dev), dev_err=err)
        kv = [kv_of(len(hist[s]), new_tok[s]) for s in seqs]
        for s, x in zip(seqs, kv):
            hist[s].append(x)
        key = torch.stack([x[0] for x in kv]).to(dev)
        val = torch.stack([x[1] for x in kv]).to(dev)
        pa.reshape_and_cache(key, val, kc, vc, torch.tensor(slots, dtype=torch.int64, device=dev), dev_err=err)
        qd = (torch.randn(len(seqs), HQ, D, generator=torch.Generator().manual_seed(100 + step))).to(torch.bfloat16)
        ctx = np.array([len(hist[s]) for s in seqs], dtype=np.int32)
        dout = torch.empty(len(seqs), HQ, D, dtype=torch.float32, device=dev)
        pa.decode(dout, qd.to(dev), kc, vc, torch.from_numpy(tables(seqs)).to(dev), torch.from_numpy(ctx).to(dev),
                  scale, partition_size=32, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        got = dout.double().cpu().numpy()
        for j, s in enumerate(seqs):
            ref = reference(qd[j].double().numpy(), hist[s], scale)
            assert np.abs(got[j] - ref).max() <= TOL, (step, s)
    # the two samples shared request 0's partly filled last block: the first
    # writer into it copied it
    assert total_copies >= 1
