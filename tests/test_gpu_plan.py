"""The decode plan's work list against a plain Python model of the same rules.

The plan kernel turns context lengths and block tables into the list of work
items the attend kernel runs ("PagedAttention blog", section 4: parallel
samples map their logical blocks to the same physical blocks, so one read of a
shared block can serve all of them).  Attend parity pins what the items
compute; this test pins the list itself, item by item: which partitions are
packed for which sequences, which shared items are split over streams, the
order (whole partitions in sequence order, then ragged tails, longest length
class first) and each item's context and split slot.  A dropped or duplicated
item, or a lost packing opportunity, fails here even where outputs would agree.
"""

import numpy as np
import pytest
import torch

from paged_kv_cache_382_b200 import workloads as W
from plan_model import model_plan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


def device_plan(pa, step, P):
    dev = "cuda"
    tables = torch.from_numpy(step.block_tables.astype(np.int32)).to(dev)
    ctx = torch.from_numpy(step.context_lens.astype(np.int32)).to(dev)
    out = torch.empty(step.num_seqs, step.num_heads, step.head_dim, dtype=torch.bfloat16, device=dev)
    cap = pa.decode_capacity(tables, step.block_size, step.max_context_len)
    ws = pa.alloc_workspace(step.num_seqs, step.num_heads, step.head_dim, cap, P, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pa.decode(out, step.q, step.k_cache, step.v_cache, tables, ctx, step.scale, partition_size=P, workspace=ws,
              max_context_len=cap, dev_err=err, phases=pa.PHASE_PLAN)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    w = ws.cpu()
    count = int(w[:4].view(torch.int32)[0])
    raw = w[256:256 + 16 * count].view(torch.int32).view(count, 4).numpy()
    return [(int(r[0]), int(r[1]), int(r[2])) for r in raw], max(1, -(-cap // P))


def check(pa, step, P):
    got, max_parts = device_plan(pa, step, P)
    want = model_plan([int(c) for c in step.context_lens], step.block_tables, P, step.block_size, step.num_heads,
                      step.num_kv_heads, max_parts)
    assert len(got) == len(want), (len(got), len(want))
    for i, (x, y) in enumerate(zip(got, want)):
        assert x == y, f"item {i}: {x} != {y}"
    return got


def test_plan_of_the_benchmark_batches(pa):
    """Private batches (every sequence its own items, tails by class) and the
    shared-prompt batches (packed and split items), at their full sizes."""
    for name, step in [("llama7b", W.llama7b(device="cuda")), ("gqa", W.gqa(device="cuda")),
                       ("long_context", W.long_context(device="cuda")),
                       ("shared_prefix", W.shared_prefix(device="cuda")),
                       ("cow", W.shared_prefix(prompt_len=520, suffix_max=0, device="cuda"))]:
        items = check(pa, step, 512)
        assert len(items) > 0, name


@pytest.mark.parametrize("seed", range(6))
def test_plan_of_random_fork_histories(pa, seed):
    """Sharing spans that end anywhere, siblings adjacent or apart."""
    from test_gpu_parity import random_fork_step

    for heads in [(16, 4), (8, 4), (8, 8), (32, 8)]:
        for adjacent in (True, False):
            for P in (32, 64):
                check(pa, random_fork_step(seed, heads[0], heads[1], 128, 16, P, adjacent), P)


@pytest.mark.parametrize("P,B,samples,prompts", [(64, 16, 6, 16), (128, 8, 8, 3), (32, 32, 24, 2),
                                                  (256, 16, 8, 200), (64, 4, 3, 400)])
def test_plan_of_shared_prompts(pa, P, B, samples, prompts):
    """Shared prompts of 1-400 prompts x 3-24 samples: runs cut at pack size and
    at chunk ends (1600 and 1200 sequences span two chunks of 1024), more
    shared units than the workspace splits, partitions of 2-128 blocks."""
    for Hq in (32, 8):
        step = W.shared_prefix(prompt_len=3 * P + 8, suffix_max=P + 5, prompts=prompts, samples=samples,
                               device="cuda", partition_size=P, num_heads=Hq, num_kv_heads=8, head_dim=128,
                               block_size=B)
        items = check(pa, step, P)
        if Hq == 32 and samples >= 3:
            assert any((x[0] & 31) > 0 for x in items), "packed items expected"
