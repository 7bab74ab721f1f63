"""The Python model of the decode plan (tests/plan_model.py) on a batch worked
out by hand; the GPU test compares the plan kernel's work list with the model."""

import numpy as np

from plan_model import model_plan


def code(s, p, count, max_parts, stream=0):
    return ((s * max_parts + p) << 7) | (stream << 5) | (count - 1)


def test_hand_worked_plan():
    """P = 32, B = 16 (two blocks per partition), 32 q / 8 kv heads (g = 4, up
    to 6 sequences per packed item), max_parts = 3.

    - sequences 0-2 share partition 0 (blocks 1, 2); 1 and 2 also partition 1
      (blocks 3, 4); sequence 3 shares nothing;
    - runs start at sequence 0 (a chain of 3) and at sequence 3;
    - partition 0 of the run 0-2 is one item of 3 sequences x 4 heads = 12
      columns (> 8): split into 3 stream items with split slot 0;
    - partition 1 of sequences 1 and 2 is not packed: only a run's first
      sequence emits shared items, and sequence 0 has no partition 1;
    - tails: 40 % 32 = 8 tokens (class 1), 70 % 32 = 6 and 65 % 32 = 1 (class
      0), sequence 3 (32 tokens) has none; the longest class comes first."""
    tables = np.array([[1, 2, 9, 10, 0], [1, 2, 3, 4, 11], [1, 2, 3, 4, 12], [5, 6, 7, 8, 13]], dtype=np.int32)
    ctx = [40, 70, 65, 32]
    mp = 3
    assert model_plan(ctx, tables, 32, 16, 32, 8, mp) == [
        (code(0, 0, 3, mp, 0), 40, 0), (code(0, 0, 3, mp, 1), 40, 0), (code(0, 0, 3, mp, 2), 40, 0),
        (code(1, 1, 1, mp), 70, -1), (code(2, 1, 1, mp), 65, -1), (code(3, 0, 1, mp), 32, -1),
        (code(0, 1, 1, mp), 40, -1), (code(1, 2, 1, mp), 70, -1), (code(2, 2, 1, mp), 65, -1),
    ]


def test_no_sharing_without_packing():
    """More than 8 query heads per kv head pack nothing: every sequence emits its
    own partitions, shared blocks or not."""
    tables = np.array([[1, 2, 3, 4], [1, 2, 3, 4]], dtype=np.int32)
    items = model_plan([64, 64], tables, 32, 16, 16, 1, 2)   # g = 16: pack 1
    assert items == [(code(0, 0, 1, 2), 64, -1), (code(0, 1, 1, 2), 64, -1),
                     (code(1, 0, 1, 2), 64, -1), (code(1, 1, 1, 2), 64, -1)]


def test_empty_context_is_a_tail_of_the_shortest_class():
    """An empty context has no whole partition and one tail item (its unit
    writes zeros) in the shortest class, after every whole partition."""
    tables = np.zeros((2, 3), dtype=np.int32)
    assert model_plan([0, 33], tables, 32, 16, 8, 8, 2) == [
        (code(1, 0, 1, 2), 33, -1), (code(0, 0, 1, 2), 0, -1), (code(1, 1, 1, 2), 33, -1)]
