"""KV utilisation: paged blocks against contiguous pre-allocation (CPU)."""

import math

import numpy as np
import pytest

from paged_kv_cache_382_b200.utilization import kv_utilisation


def test_worked_example():
    # the blog's 7-token prompt at B = 4 holds 7 of 8 paged slots; pre-allocated
    # to a 2048-token maximum it holds 7 of 2048
    u = kv_utilisation([7], block_size=4, max_len=2048)
    assert u["paged_slots"] == 8 and u["paged"] == 7 / 8
    assert u["contiguous_slots"] == 2048 and u["contiguous"] == 7 / 2048


def test_paged_waste_is_below_one_block_per_sequence():
    rng = np.random.default_rng(0)
    ctx = rng.integers(1, 5000, size=500)
    for B in (4, 8, 16, 32):
        u = kv_utilisation(ctx, B, 8192)
        assert u["paged_slots"] - u["tokens"] < B * len(ctx)
        assert u["paged"] > u["contiguous"]


def test_gqa_length_distribution():
    """The GQA workload's log-normal lengths (median 1000, capped at 8192): a
    contiguous reservation of the cap holds well under half its slots, paged
    blocks of 16 hold more than 99 %."""
    rng = np.random.default_rng(0)
    ctx = np.clip(np.round(np.exp(math.log(1000.0) + rng.standard_normal(256))), 1, 8192)
    u = kv_utilisation(ctx, 16, 8192)
    assert u["contiguous"] < 0.4 and u["paged"] > 0.99


def test_rejects_lengths_beyond_max():
    with pytest.raises(ValueError):
        kv_utilisation([10, 3000], 16, 2048)
