"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Bars, from the decode-attention target: scatter and block copies bit-exact;
decode max |err| <= 1e-5 for fp32 inputs and <= 2e-3 for bf16 inputs with fp32
accumulation (fp32 output); a bf16 output may differ by a further half bf16 ulp
of the exact value, the rounding of the output itself.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_382_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5
TOL_BF16 = 2e-3


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

class SparsePool:
    """Some blocks of a pool, indexed by physical id like the full array.

    Lets the oracle run on the blocks one sequence touches without copying a
    multi-gigabyte pool to the host."""

    def __init__(self, blocks, shape):
        self.blocks = blocks
        self.shape = shape

    @classmethod
    def fetch(cls, pool: torch.Tensor, ids, as_float=True):
        ids = sorted(set(int(i) for i in ids))
        idx = torch.tensor(ids, dtype=torch.long, device=pool.device)
        rows = pool.index_select(0, idx)
        rows = rows.to("cpu", torch.float64).numpy() if as_float else raw_bits(rows)
        return cls({b: rows[i].copy() for i, b in enumerate(ids)}, tuple(pool.shape))

    def copy(self):
        return SparsePool({k: v.copy() for k, v in self.blocks.items()}, self.shape)

    def __getitem__(self, idx):
        if isinstance(idx, tuple):
            return self.blocks[int(idx[0])][idx[1:]]
        return self.blocks[int(idx)]

    def __setitem__(self, idx, val):
        if isinstance(idx, tuple):
            self.blocks[int(idx[0])][idx[1:]] = val
        else:
            self.blocks[int(idx)] = np.array(val, copy=True)


def raw_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32).numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def to_device(step: W.DecodeStep, device="cuda") -> W.DecodeStep:
    for name in ("q", "k_cache", "v_cache", "new_key", "new_value"):
        setattr(step, name, getattr(step, name).to(device))
    return step


def run_gpu(pa, step, out_dtype=torch.float32, partition_size=None, max_context_len=0,
            keep_pre=False, tables=None, slots=None, pairs=None, ctx=None):
    dev = "cuda"
    pre = (step.k_cache.clone(), step.v_cache.clone()) if keep_pre else None
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pairs = step.copy_pairs if pairs is None else pairs
    if len(pairs):
        pa.copy_blocks(kc, vc, torch.from_numpy(np.ascontiguousarray(pairs)).to(dev), dev_err=err)
    slots = step.slot_mapping if slots is None else slots
    if len(slots):
        pa.reshape_and_cache(step.new_key, step.new_value, kc, vc, torch.from_numpy(slots).to(dev),
                             dev_err=err)
    tables = step.block_tables if tables is None else tables
    ctx = step.context_lens if ctx is None else ctx
    out = torch.empty(step.num_seqs, step.num_heads, step.head_dim, dtype=out_dtype, device=dev)
    pa.decode(out, step.q, kc, vc, torch.from_numpy(np.ascontiguousarray(tables, dtype=np.int32)).to(dev),
              torch.from_numpy(np.ascontiguousarray(ctx, dtype=np.int32)).to(dev), step.scale,
              partition_size=partition_size or step.partition_size, max_context_len=max_context_len,
              dev_err=err)
    torch.cuda.synchronize()
    return out, kc, vc, int(err.item()), pre


def oracle_outputs(step, seqs, pre_k, pre_v):
    """Oracle output rows for the given sequences, from the pool as it was before
    this step's copies and writes (pre_k / pre_v on the device)."""
    res = {}
    B = step.block_size
    for s in seqs:
        c = int(step.context_lens[s])
        table = step.block_tables[s]
        blocks = [int(b) for b in table[: -(-c // B)]]
        pairs = [(int(a), int(b)) for a, b in step.copy_pairs if int(b) in blocks]
        need = set(blocks) | {a for a, _ in pairs}
        if not need:
            res[s] = np.zeros((step.num_heads, step.head_dim))
            continue
        kp = SparsePool.fetch(pre_k, need)
        vp = SparsePool.fetch(pre_v, need)
        kp, vp = oracle.copy_blocks(kp, vp, pairs)
        # this sequence's token of the step is row s of the step's writes
        mine = [t for t in range(len(step.slot_mapping)) if t == s and step.slot_mapping[t] >= 0]
        if mine:
            t = mine[0]
            kp, vp = oracle.reshape_and_cache(f64(step.new_key[t:t + 1]), f64(step.new_value[t:t + 1]),
                                              kp, vp, step.slot_mapping[t:t + 1])
        res[s] = oracle.decode_attention(f64(step.q[s:s + 1]), kp, vp, table[None], np.array([c]),
                                         step.scale)[0]
    return res


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 8), 0.0)


def assert_close(got, ref, dtype_in, out_dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    tol = TOL_F32 if dtype_in == torch.float32 else TOL_BF16
    bound = tol + (bf16_half_ulp(ref) if out_dtype == torch.bfloat16 else 0.0)
    worst = float((err - bound).max())
    assert worst <= 0.0, f"{what}: max |err| {float(err.max()):.3e} exceeds the bound by {worst:.3e}"
    return float(err.max())


# ---------------------------------------------------------------------------
# small cases: every output row against the oracle
# ---------------------------------------------------------------------------

def full_oracle(step):
    kc, vc = f64(step.k_cache), f64(step.v_cache)
    kc, vc = oracle.copy_blocks(kc, vc, step.copy_pairs)
    kc, vc = oracle.reshape_and_cache(f64(step.new_key), f64(step.new_value), kc, vc, step.slot_mapping)
    return oracle.decode_attention(f64(step.q), kc, vc, step.block_tables, step.context_lens, step.scale)


@pytest.mark.parametrize("block_size", [16, 4])
@pytest.mark.parametrize("partition_size", [512, 32])
def test_tiny_fp32(pa, block_size, partition_size):
    step = to_device(W.tiny(block_size=block_size, poison=True))
    out, *_ = run_gpu(pa, step, partition_size=partition_size)
    err = assert_close(f64(out), full_oracle(step), torch.float32, torch.float32, "tiny fp32")
    assert err < TOL_F32


SMALL_BF16 = [
    # (ctx lens, Hq, Hkv, d, B, P)
    ([7, 16, 33, 100], 4, 4, 64, 16, 512),
    ([7, 16, 33, 100], 4, 4, 64, 4, 32),
    ([1, 2, 15, 16, 17, 31, 33, 257], 8, 2, 128, 16, 64),
    ([0, 5, 300, 1000], 32, 8, 128, 16, 512),
    ([0, 5, 300, 1000], 32, 8, 128, 8, 128),
    ([1, 40, 613, 1024, 1025], 64, 8, 128, 32, 512),
    ([129, 3, 77], 16, 1, 128, 16, 32),
    ([50, 513, 9], 6, 2, 64, 8, 64),
    ([700, 1], 12, 1, 64, 4, 96),
    ([2049, 64], 8, 8, 128, 32, 8192),
]


@pytest.mark.parametrize("case", SMALL_BF16, ids=lambda c: f"ctx{len(c[0])}_h{c[1]}x{c[2]}_d{c[3]}_b{c[4]}_p{c[5]}")
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32out", "bf16out"])
def test_small_bf16(pa, case, out_dtype):
    ctx, Hq, Hkv, d, B, P = case
    step = to_device(W.independent("small", ctx, dtype=torch.bfloat16, num_heads=Hq, num_kv_heads=Hkv,
                                   head_dim=d, block_size=B, seed=len(ctx) + Hq + B, poison=True,
                                   partition_size=P))
    out, _, _, err, _ = run_gpu(pa, step, out_dtype=out_dtype)
    assert err == 0
    assert_close(f64(out), full_oracle(step), torch.bfloat16, out_dtype, str(case))


def test_many_sequences_plan_chunks(pa):
    """More sequences than the plan kernel's 1024 threads, lengths 0..40."""
    rng = np.random.default_rng(11)
    ctx = rng.integers(0, 41, size=3000)
    step = to_device(W.independent("many", ctx, dtype=torch.bfloat16, num_heads=8, num_kv_heads=2,
                                   head_dim=64, block_size=8, seed=3, partition_size=32))
    out, _, _, err, _ = run_gpu(pa, step)
    assert err == 0
    ref = full_oracle(step)
    assert_close(f64(out), ref, torch.bfloat16, torch.float32, "many sequences")


# ---------------------------------------------------------------------------
# the cache writes: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_reshape_and_cache_bit_exact_small(pa, dtype):
    step = to_device(W.independent("w", [1, 4, 5, 0, 33, 16, 17], dtype=dtype, num_heads=4, num_kv_heads=4,
                                   head_dim=64 if dtype == torch.float32 else 128, block_size=4, seed=5))
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    pa.reshape_and_cache(step.new_key, step.new_value, kc, vc, torch.from_numpy(step.slot_mapping).cuda())
    torch.cuda.synchronize()
    ek, ev = oracle.reshape_and_cache(raw_bits(step.new_key), raw_bits(step.new_value),
                                      raw_bits(step.k_cache), raw_bits(step.v_cache), step.slot_mapping)
    assert np.array_equal(raw_bits(kc), ek) and np.array_equal(raw_bits(vc), ev)


def test_copy_blocks_bit_exact_small(pa):
    step = to_device(W.shared_prefix(prompt_len=520, suffix_max=0, prompts=2, samples=4))
    assert len(step.copy_pairs) == 2 * 3
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    pa.copy_blocks(kc, vc, torch.from_numpy(step.copy_pairs).cuda())
    torch.cuda.synchronize()
    ek, ev = oracle.copy_blocks(raw_bits(step.k_cache), raw_bits(step.v_cache), step.copy_pairs)
    assert np.array_equal(raw_bits(kc), ek) and np.array_equal(raw_bits(vc), ev)


# ---------------------------------------------------------------------------
# full-size workloads, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------

FULL = {
    "llama7b": lambda: W.llama7b(device="cuda"),
    "gqa": lambda: W.gqa(device="cuda"),
    "shared_prefix_p512": lambda: W.shared_prefix(prompt_len=512, suffix_max=512, device="cuda"),
    "shared_prefix_p520_cow": lambda: W.shared_prefix(prompt_len=520, suffix_max=0, device="cuda"),
    "shared_prefix_p512_part256": lambda: W.shared_prefix(prompt_len=512, suffix_max=512, device="cuda",
                                                          partition_size=256),
    "long_context_b8": lambda: W.long_context(block_size=8, device="cuda"),
    "long_context_b16": lambda: W.long_context(block_size=16, device="cuda"),
    "long_context_b32": lambda: W.long_context(block_size=32, device="cuda"),
}


def run_fused_step(pa, step, out_dtype):
    """The benchmark's launch configuration: one pa_decode_step call with the
    capacity bound, workspace and output dtype bench.py uses."""
    dev = "cuda"
    pre = (step.k_cache.clone(), step.v_cache.clone())
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    tables = torch.from_numpy(step.block_tables.astype(np.int32)).to(dev)
    cap = pa.decode_capacity(tables, step.block_size, step.max_context_len)
    ws = pa.alloc_workspace(step.num_seqs, step.num_heads, step.head_dim, cap, step.partition_size, dev)
    out = torch.empty(step.num_seqs, step.num_heads, step.head_dim, dtype=out_dtype, device=dev)
    pairs = torch.from_numpy(np.ascontiguousarray(step.copy_pairs)).to(dev) if len(step.copy_pairs) else None
    pa.decode_step(out, step.q, step.new_key, step.new_value, kc, vc, torch.from_numpy(step.slot_mapping).to(dev),
                   tables, torch.from_numpy(step.context_lens.astype(np.int32)).to(dev), step.scale,
                   copy_pairs=pairs, max_context_len=cap, partition_size=step.partition_size, workspace=ws,
                   dev_err=err)
    torch.cuda.synchronize()
    return out, kc, vc, int(err.item()), pre


@pytest.mark.parametrize("call", ["phased", "fused_step_bf16_out"])
@pytest.mark.parametrize("name", list(FULL))
def test_full_size(pa, name, call):
    step = FULL[name]()
    if call == "phased":
        out_dtype = torch.float32
        out, kc, vc, err, pre = run_gpu(pa, step, keep_pre=True)
    else:
        out_dtype = torch.bfloat16
        out, kc, vc, err, pre = run_fused_step(pa, step, out_dtype)
    assert err == 0
    assert torch.isfinite(out).all()
    pre_k, pre_v = pre
    # cache writes: every touched block bit-exact, every other block untouched
    touched = sorted({int(s) // step.block_size for s in step.slot_mapping if s >= 0}
                     | {int(b) for _, b in step.copy_pairs})
    srcs = {int(a) for a, _ in step.copy_pairs}
    kp = SparsePool.fetch(pre_k, set(touched) | srcs, as_float=False)
    vp = SparsePool.fetch(pre_v, set(touched) | srcs, as_float=False)
    kp, vp = oracle.copy_blocks(kp, vp, step.copy_pairs)
    kp, vp = oracle.reshape_and_cache(raw_bits(step.new_key), raw_bits(step.new_value), kp, vp,
                                      step.slot_mapping)
    idx = torch.tensor(touched, dtype=torch.long, device="cuda")
    got_k, got_v = raw_bits(kc.index_select(0, idx)), raw_bits(vc.index_select(0, idx))
    for i, b in enumerate(touched):
        assert np.array_equal(got_k[i], kp[b]) and np.array_equal(got_v[i], vp[b]), f"block {b}"
    untouched = torch.ones(step.num_blocks, dtype=torch.bool, device="cuda")
    untouched[idx] = False
    assert torch.equal(kc[untouched], pre_k[untouched]) and torch.equal(vc[untouched], pre_v[untouched])
    # decode: every sequence, every head, against the oracle run one sequence at
    # a time on the blocks it reads (the oracle redoes the step's copies and write)
    ctx = step.context_lens
    seqs = list(range(step.num_seqs))
    ref = oracle_outputs(step, seqs, pre_k, pre_v)
    got = f64(out)
    for s in seqs:
        assert_close(got[s], ref[s], torch.bfloat16, out_dtype, f"{name} seq {s} ctx {ctx[s]}")


# ---------------------------------------------------------------------------
# invariants the pages fix, checked bit for bit on the GPU
# ---------------------------------------------------------------------------

def test_reservation_and_free_blocks_are_ignored(pa):
    """NaN in every free block and reservation slot, -1 past each table's end:
    the output equals the run without them, bit for bit, and is finite."""
    kw = dict(dtype=torch.bfloat16, num_heads=16, num_kv_heads=4, head_dim=128, block_size=16, seed=21,
              partition_size=64)
    ctx = [1, 17, 100, 333, 64, 65]
    clean = to_device(W.independent("clean", ctx, poison=False, **kw))
    dirty = to_device(W.independent("dirty", ctx, poison=True, **kw))
    a, *_ = run_gpu(pa, clean)
    b, *_ = run_gpu(pa, dirty)
    assert torch.isfinite(b).all()
    assert torch.equal(a, b)


def test_permutation_of_physical_blocks(pa):
    step = to_device(W.independent("perm", [3, 95, 640, 17, 1100], dtype=torch.bfloat16, num_heads=32,
                                   num_kv_heads=8, head_dim=128, block_size=16, seed=9, partition_size=128))
    base, *_ = run_gpu(pa, step)
    perm = np.random.default_rng(5).permutation(step.num_blocks)
    inv = torch.from_numpy(np.argsort(perm)).cuda()
    moved = W.DecodeStep(**{**step.__dict__})
    moved.k_cache = step.k_cache[inv].contiguous()    # block b moves to perm[b]
    moved.v_cache = step.v_cache[inv].contiguous()
    moved.block_tables = np.where(step.block_tables >= 0, perm[np.maximum(step.block_tables, 0)], -1)
    moved.slot_mapping = np.where(step.slot_mapping >= 0,
                                  perm[step.slot_mapping // step.block_size] * step.block_size
                                  + step.slot_mapping % step.block_size, -1)
    again, *_ = run_gpu(pa, moved)
    assert torch.equal(base, again)


def test_deterministic_and_shared_tables(pa):
    step = to_device(W.independent("det", [900, 900, 31], dtype=torch.bfloat16, num_heads=32,
                                   num_kv_heads=8, head_dim=128, block_size=16, seed=4, partition_size=256))
    step.q[1] = step.q[0]
    tables = step.block_tables.copy()
    tables[1] = tables[0]                  # sequence 1 reads sequence 0's blocks
    slots = step.slot_mapping.copy()
    slots[1] = -1                           # ... and writes nothing of its own
    a, *_ = run_gpu(pa, step, tables=tables, slots=slots)
    b, *_ = run_gpu(pa, step, tables=tables, slots=slots)
    assert torch.equal(a, b)
    assert torch.equal(a[0], a[1])


def test_attend_phases_repeat_over_one_plan(pa):
    """Units are handed out by a ticket that the plan resets and each attend
    launch's last fetch puts back: attend + reduce run twice over one plan give
    the result of the whole call, bit for bit, both times (many more units
    than CTAs)."""
    step = to_device(W.independent("phases", [2000] * 96 + [17] * 64, dtype=torch.bfloat16, num_heads=32,
                                   num_kv_heads=8, head_dim=128, block_size=16, seed=8, partition_size=128))
    ref, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    tables = torch.from_numpy(step.block_tables.astype(np.int32)).cuda()
    ctx = torch.from_numpy(step.context_lens.astype(np.int32)).cuda()
    ws = pa.alloc_workspace(step.num_seqs, step.num_heads, step.head_dim,
                            pa.decode_capacity(tables, step.block_size, 0), step.partition_size, "cuda")
    kw = dict(partition_size=step.partition_size, workspace=ws)
    pa.decode(torch.empty_like(ref), step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_PLAN, **kw)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        pa.decode(out, step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_ATTEND, **kw)
        pa.decode(out, step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_REDUCE, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def unshared_copy(step):
    """The same batch with every sequence's blocks copied to private physical
    blocks: identical contents, no shared block ids, hence no packed units."""
    B = step.block_size
    ids, tables = [], np.full_like(step.block_tables, -1)
    for sq in range(step.num_seqs):
        nb = -(-int(step.context_lens[sq]) // B)
        tables[sq, :nb] = np.arange(len(ids), len(ids) + nb)
        ids.extend(int(b) for b in step.block_tables[sq, :nb])
    idx = torch.tensor(ids, dtype=torch.long, device=step.k_cache.device)
    out = W.DecodeStep(**{**step.__dict__})
    out.k_cache = step.k_cache.index_select(0, idx).contiguous()
    out.v_cache = step.v_cache.index_select(0, idx).contiguous()
    out.num_blocks = len(ids)
    out.block_tables = tables
    out.slot_mapping = np.full_like(step.slot_mapping, -1)   # pools are compared after the step's writes
    out.copy_pairs = np.zeros((0, 2), dtype=np.int64)
    return out


@pytest.mark.parametrize("heads", [(32, 8), (16, 8), (8, 8)], ids=["g4", "g2", "g1"])
def test_packed_shared_prefix_units_are_bit_identical(pa, heads):
    """Samples that share a prompt's blocks are served by packed units; the
    result equals, bit for bit, the same batch with private copies of the blocks
    (and the oracle)."""
    Hq, Hkv = heads
    step = W.shared_prefix(prompt_len=96, suffix_max=50, prompts=3, samples=5, device="cuda",
                           partition_size=32, num_heads=Hq, num_kv_heads=Hkv, head_dim=128, block_size=16)
    out, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    after = W.DecodeStep(**{**step.__dict__})
    after.k_cache, after.v_cache = kc, vc          # the pool after this step's copies and writes
    plain = unshared_copy(after)
    out2, *_ = run_gpu(pa, plain)
    assert torch.equal(out, out2)
    assert_close(f64(out), full_oracle(step), torch.bfloat16, torch.float32, f"packed {heads}")


SHARED_LAYOUTS = [
    # (Hq, Hkv, samples): query columns per shared unit = samples x g, in column groups of 8
    (32, 8, 8),    # g 4: 32 columns, 4 groups
    (32, 8, 5),    # 20 columns, 3 groups
    (32, 8, 3),    # 12 columns, 2 groups
    (16, 8, 12),   # g 2: 24 columns
    (8, 8, 32),    # g 1: 32 columns
    (8, 8, 12),    # 12 columns
    (64, 8, 4),    # g 8: 32 columns
    (64, 8, 3),    # 24 columns
    (24, 8, 7),    # g 3: 21 columns, sequences straddle column groups
]


@pytest.mark.parametrize("d,B,P", [(128, 16, 128), (64, 8, 64), (128, 32, 32)], ids=["d128_b16_p128", "d64_b8_p64",
                                                                                    "d128_b32_p32"])
@pytest.mark.parametrize("layout", SHARED_LAYOUTS, ids=lambda c: f"h{c[0]}x{c[1]}_s{c[2]}")
def test_shared_units_of_every_width(pa, layout, d, B, P):
    """Samples sharing whole partitions are served by units of up to 32 query
    columns that read each shared tile once (one warp per column group, a ring
    of tiles shared by the CTA).  The output equals, bit for bit, the same batch
    with private copies of the blocks (units of one column group, each warp one
    stream), and the oracle within tolerance."""
    Hq, Hkv, samples = layout
    step = W.shared_prefix(prompt_len=3 * P + 8, suffix_max=P + 5, prompts=2, samples=samples, device="cuda",
                           partition_size=P, num_heads=Hq, num_kv_heads=Hkv, head_dim=d, block_size=B)
    out, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    after = W.DecodeStep(**{**step.__dict__})
    after.k_cache, after.v_cache = kc, vc
    out2, *_ = run_gpu(pa, unshared_copy(after))
    assert torch.equal(out, out2)
    assert_close(f64(out), full_oracle(step), torch.bfloat16, torch.float32, f"shared {layout}")


def test_shared_units_beyond_the_split_capacity(pa):
    """More shared partitions than the workspace holds split units for (256 units
    of one kv head): the first ones run as W stream units on different CTAs,
    merged by the last, the rest as one CTA; all bit-identical to private copies
    and within tolerance of the oracle."""
    step = W.shared_prefix(prompt_len=64 * 3, suffix_max=20, prompts=16, samples=6, device="cuda",
                           partition_size=64, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16)
    # 16 prompts x 3 shared partitions = 48 shared items x 8 kv heads = 384 units > 256
    out, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    after = W.DecodeStep(**{**step.__dict__})
    after.k_cache, after.v_cache = kc, vc
    out2, *_ = run_gpu(pa, unshared_copy(after))
    assert torch.equal(out, out2)
    assert_close(f64(out), full_oracle(step), torch.bfloat16, torch.float32, "beyond the split capacity")


def test_split_units_repeat_over_one_plan(pa):
    """Split shared units count their finished streams in the workspace; the last
    one resets the count, so attend + reduce run twice over one plan give the
    whole call's result bit for bit both times."""
    step = W.shared_prefix(prompt_len=300, suffix_max=60, prompts=4, samples=8, device="cuda", partition_size=128,
                           num_heads=32, num_kv_heads=8, head_dim=128, block_size=16)
    ref, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    tables = torch.from_numpy(step.block_tables.astype(np.int32)).cuda()
    ctx = torch.from_numpy(step.context_lens.astype(np.int32)).cuda()
    ws = pa.alloc_workspace(step.num_seqs, step.num_heads, step.head_dim,
                            pa.decode_capacity(tables, step.block_size, 0), step.partition_size, "cuda")
    kw = dict(partition_size=step.partition_size, workspace=ws)
    pa.decode(torch.empty_like(ref), step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_PLAN, **kw)
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        pa.decode(out, step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_ATTEND, **kw)
        pa.decode(out, step.q, kc, vc, tables, ctx, step.scale, phases=pa.PHASE_REDUCE, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_bad_block_in_a_shared_partition(pa):
    """A block id outside the pool inside a shared partition: flagged, its tokens
    skipped by every sample (their value rows zeroed by the ring's issuer), and
    the result equals, bit for bit, private copies with the same bad entry."""
    step = W.shared_prefix(prompt_len=200, suffix_max=40, prompts=2, samples=8, device="cuda", partition_size=64,
                           num_heads=32, num_kv_heads=8, head_dim=128, block_size=16)
    out_ok, kc, vc, err, _ = run_gpu(pa, step)
    assert err == 0
    after = W.DecodeStep(**{**step.__dict__})
    after.k_cache, after.v_cache = kc, vc
    after.slot_mapping = np.full_like(step.slot_mapping, -1)
    after.copy_pairs = np.zeros((0, 2), dtype=np.int64)
    plain = unshared_copy(after)
    bad = after.num_blocks + 3
    shared_tables = after.block_tables.copy()
    shared_tables[:, 5] = bad                  # logical block 5: inside the shared second partition
    plain_tables = plain.block_tables.copy()
    plain_tables[:, 5] = bad + plain.num_blocks
    a, _, _, ea, _ = run_gpu(pa, after, tables=shared_tables)
    b, _, _, eb, _ = run_gpu(pa, plain, tables=plain_tables)
    assert ea & pa.DEVERR_BLOCK_ID and eb & pa.DEVERR_BLOCK_ID
    assert torch.isfinite(a).all()
    assert torch.equal(a, b)
    assert not torch.equal(a, out_ok)


def random_fork_step(seed, Hq, Hkv, d, B, P, adjacent=True):
    """A batch whose block tables come from a random serving history through the
    block manager: prompts, forks at random points (a child shares every block
    of its parent up to the fork, then diverges, mid-block included) and ragged
    appends.  Children sit next to their parents (packing applies) unless
    `adjacent` is false.  The pool holds random values in every block."""
    from paged_kv_cache_382_b200.blocks import BlockManager, BlockPool, block_table_array

    rng = np.random.default_rng(seed)
    NB = 600
    mgr = BlockManager(BlockPool(NB, rng.permutation(NB)), B)
    seqs = []
    for _ in range(3):                       # prompts
        sq = mgr.new_sequence()
        mgr.append_tokens(sq, int(rng.integers(1, 200)))
        seqs.append(sq)
    for _ in range(12):                      # forks with their own continuations
        i = int(rng.integers(0, len(seqs)))
        child = mgr.fork(seqs[i])
        mgr.append_tokens(child, int(rng.integers(0, 90)))
        seqs.insert(i + 1 if adjacent else len(seqs), child)
    for sq in seqs:                          # every sequence gets this step's token
        mgr.append_tokens(sq, 1)
    gen = torch.Generator(device="cuda").manual_seed(seed)
    normal = lambda *shape: torch.empty(*shape, dtype=torch.float32, device="cuda").normal_(generator=gen).to(
        torch.bfloat16)  # noqa: E731
    S = len(seqs)
    return W.DecodeStep(
        name=f"random_fork_{seed}", dtype=torch.bfloat16, num_heads=Hq, num_kv_heads=Hkv, head_dim=d, block_size=B,
        num_blocks=NB, context_lens=np.array([sq.num_tokens for sq in seqs], dtype=np.int32),
        block_tables=block_table_array(seqs), scale=float(np.float32(1.0 / math.sqrt(d))), partition_size=P,
        q=normal(S, Hq, d), k_cache=normal(NB, Hkv, B, d), v_cache=normal(NB, Hkv, B, d),
        new_key=normal(S, Hkv, d), new_value=normal(S, Hkv, d),
        slot_mapping=np.full(S, -1, dtype=np.int64), copy_pairs=np.zeros((0, 2), dtype=np.int64))


@pytest.mark.parametrize("heads,B", [((32, 8), 16), ((8, 8), 4), ((64, 8), 8)], ids=["g4_b16", "g1_b4", "g8_b8"])
def test_short_tails_and_batch_order(pa, heads, B):
    """Ragged tails of every length class, single-tile ones and empty contexts
    included, at block sizes 16, 4 and 8: against the oracle, and independent
    of the batch around them: the batch reversed, and with one sequence dropped
    (other units around each tail, other unit counts per class), gives every
    remaining row bit for bit."""
    Hq, Hkv = heads
    P = 64
    rng = np.random.default_rng(11)
    rests = [0, 1, 5, 9, 16, 17, 30, 63]
    ctx = [int(P * rng.integers(0, 4) + rests[i % len(rests)]) for i in range(26)]
    ctx[3] = 0
    step = W.independent("single_tile_tails", ctx, num_heads=Hq, num_kv_heads=Hkv, block_size=B, seed=5,
                         device="cuda", partition_size=P)
    out, *_, err, _ = run_gpu(pa, step, out_dtype=torch.bfloat16)
    assert err == 0
    assert_close(f64(out), full_oracle(step), torch.bfloat16, torch.bfloat16, "single-tile tails")
    S = step.num_seqs
    for order in (list(range(S - 1, -1, -1)), [i for i in range(S) if i != 7]):
        other = W.DecodeStep(**{**step.__dict__})
        other.q = step.q[order].contiguous()
        other.block_tables = step.block_tables[order]
        other.context_lens = step.context_lens[order]
        other.slot_mapping = step.slot_mapping[order]
        other.new_key = step.new_key[order].contiguous()
        other.new_value = step.new_value[order].contiguous()
        out2, *_, err2, _ = run_gpu(pa, other, out_dtype=torch.bfloat16)
        assert err2 == 0
        assert torch.equal(out2, out[order])


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("heads", [(16, 4), (8, 4), (8, 8)], ids=["g4", "g2", "g1"])
def test_random_fork_histories(pa, seed, heads):
    """Random sharing patterns (shared spans ending anywhere, packed runs of every
    length, siblings adjacent or not): equal to the oracle, and bit for bit to the
    same batch without shared block ids."""
    Hq, Hkv = heads
    for adjacent in (True, False):
        step = random_fork_step(seed, Hq, Hkv, 128, 16, 32, adjacent)
        out, *_, err, _ = run_gpu(pa, step)
        assert err == 0
        assert_close(f64(out), full_oracle(step), torch.bfloat16, torch.float32, f"seed {seed} {heads} {adjacent}")
        out2, *_ = run_gpu(pa, unshared_copy(step))
        assert torch.equal(out, out2)


@pytest.mark.parametrize("name", ["independent", "cow", "poisoned", "no_new_tokens"])
def test_decode_step_equals_the_three_calls(pa, name):
    """pa_decode_step (copies, scatter fused with the plan, attention, merge) gives
    bit for bit the pools and output of pa_copy_blocks, pa_reshape_and_cache and
    pa_decode called in that order."""
    kw = dict(num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, partition_size=64, device="cuda")
    if name == "cow":
        step = W.shared_prefix(prompt_len=40, suffix_max=0, prompts=3, samples=4, **kw)
    else:
        step = to_device(W.independent(name, [5, 70, 300, 1, 129, 1000], dtype=torch.bfloat16, seed=12,
                                       poison=(name == "poisoned"), **{k: v for k, v in kw.items()
                                                                        if k != "device"}))
    slots = step.slot_mapping if name != "no_new_tokens" else np.zeros(0, dtype=np.int64)
    ref_out, ref_k, ref_v, ref_err, _ = run_gpu(pa, step, slots=slots)
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(ref_out)
    T = len(slots)
    pairs = torch.from_numpy(np.ascontiguousarray(step.copy_pairs)).cuda() if len(step.copy_pairs) else None
    pa.decode_step(out, step.q, step.new_key[:T], step.new_value[:T], kc, vc, torch.from_numpy(slots).cuda(),
                   torch.from_numpy(step.block_tables).cuda(), torch.from_numpy(step.context_lens).cuda(), step.scale,
                   copy_pairs=pairs, partition_size=step.partition_size, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == ref_err
    assert torch.equal(out, ref_out)
    assert torch.equal(kc.view(torch.int16), ref_k.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), ref_v.view(torch.int16))


def test_bounded_wait_gives_up_and_the_context_survives(pa):
    """The bounded wait all asynchronous-copy waits use: a barrier nothing arrives
    at is given up on after the limit, PA_DEVERR_TIMEOUT is raised, the kernel
    returns, and the context keeps working (a decode step afterwards is exact)."""
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.selftest_bounded_wait(err, limit_ns=2_000_000)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.DEVERR_TIMEOUT
    step = to_device(W.tiny(block_size=16, poison=True))
    out, *_, e, _ = run_gpu(pa, step)
    assert e == 0
    err_max = float(np.abs(f64(out) - full_oracle(step)).max())
    assert err_max < TOL_F32


def test_single_token_context_returns_the_value_row(pa):
    step = to_device(W.independent("one", [1, 1, 1], dtype=torch.bfloat16, num_heads=8, num_kv_heads=2,
                                   head_dim=128, block_size=8, seed=2))
    out, kc, vc, _, _ = run_gpu(pa, step)
    for s in range(3):
        for h in range(8):
            assert torch.equal(out[s, h], step.new_value[s, h // 4].float())


# ---------------------------------------------------------------------------
# data-dependent errors: skipped and reported, never a fault
# ---------------------------------------------------------------------------

def test_bad_block_id_is_flagged(pa):
    step = to_device(W.independent("badblk", [40, 40], dtype=torch.bfloat16, num_heads=8, num_kv_heads=8,
                                   head_dim=128, block_size=16, seed=6))
    tables = step.block_tables.copy()
    tables[0, 1] = step.num_blocks + 5
    out, _, _, err, _ = run_gpu(pa, step, tables=tables)
    assert err & pa.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    ref = full_oracle(step)
    assert_close(f64(out[1]), ref[1], torch.bfloat16, torch.float32, "healthy sequence")


def test_bad_block_id_fp32(pa):
    step = to_device(W.tiny(block_size=4))
    tables = step.block_tables.copy()
    tables[3, 2] = -7
    out, _, _, err, _ = run_gpu(pa, step, tables=tables)
    assert err & pa.DEVERR_BLOCK_ID


def test_bad_slot_and_pair_are_flagged(pa):
    step = to_device(W.independent("badslot", [5, 9], dtype=torch.bfloat16, num_heads=4, num_kv_heads=4,
                                   head_dim=64, block_size=4, seed=8))
    slots = step.slot_mapping.copy()
    slots[0] = step.num_blocks * step.block_size + 3
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.reshape_and_cache(step.new_key, step.new_value, kc, vc, torch.from_numpy(slots).cuda(), dev_err=err)
    pa.copy_blocks(kc, vc, torch.tensor([[0, step.num_blocks]], dtype=torch.int64, device="cuda"), dev_err=err)
    torch.cuda.synchronize()
    assert err.item() & pa.DEVERR_SLOT and err.item() & pa.DEVERR_COPY
    # the valid token was still written, the invalid one and the bad copy were skipped
    ek, _ = oracle.reshape_and_cache(raw_bits(step.new_key[1:]), raw_bits(step.new_value[1:]),
                                     raw_bits(step.k_cache), raw_bits(step.v_cache), slots[1:])
    assert np.array_equal(raw_bits(kc), ek)


def test_context_above_capacity_is_clamped_and_flagged(pa):
    step = to_device(W.independent("cap", [100, 20], dtype=torch.bfloat16, num_heads=8, num_kv_heads=8,
                                   head_dim=128, block_size=16, seed=12))
    out, _, _, err, _ = run_gpu(pa, step, max_context_len=64)
    assert err & pa.DEVERR_CONTEXT
    clamped = W.DecodeStep(**{**step.__dict__})
    clamped.context_lens = np.minimum(step.context_lens, 64)
    ref = full_oracle(clamped)
    assert_close(f64(out), ref, torch.bfloat16, torch.float32, "clamped")


# ---------------------------------------------------------------------------
# prefill: a chunk of new tokens attends causally to the paged context
# ---------------------------------------------------------------------------

PREFILL_CASES = [
    # (context lens, new tokens, Hq, Hkv, d, B, P)
    ([7, 40, 100], [7, 3, 33], 4, 4, 64, 16, 32),
    ([300, 1029, 64, 1], [300, 45, 64, 1], 32, 8, 128, 16, 128),
    ([257, 600], [120, 600], 8, 8, 128, 8, 64),
    ([90, 2049], [17, 31], 16, 2, 128, 32, 512),
    ([513, 80], [9, 80], 64, 8, 64, 4, 32),
    ([200, 77, 1], [200, 20, 1], 12, 4, 128, 16, 64),     # group 3: no tensor-core tile
    ([333, 64, 129], [100, 64, 129], 32, 2, 64, 8, 128),  # group 16: 8 tokens per tile
    ([77, 40, 300], [13, 0, 37], 64, 2, 64, 16, 64),      # group 32: 4 tokens per tile; an empty sequence
    ([50, 33], [9, 33], 128, 1, 64, 32, 32),              # group 128: one token per tile
]


def prefill_inputs(case, dtype, poison=False, seed_q=7):
    ctx, new, Hq, Hkv, d, B, P = case
    step = to_device(W.independent("prefill", ctx, dtype=dtype, num_heads=Hq, num_kv_heads=Hkv, head_dim=d,
                                   block_size=B, seed=sum(new), poison=poison, partition_size=P))
    gen = torch.Generator(device="cuda").manual_seed(seed_q)
    T = sum(new)
    q = torch.empty(T, Hq, d, dtype=torch.float32, device="cuda").normal_(generator=gen).to(dtype)
    qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    return step, q, qs


def run_prefill(pa, step, q, qs, tables=None, ctx=None, out_dtype=torch.float32, max_context_len=0):
    T, Hq, d = q.shape
    out = torch.full((T, Hq, d), float("nan"), dtype=out_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = step.block_tables if tables is None else tables
    ctx = step.context_lens if ctx is None else ctx
    pa.prefill(out, q, step.k_cache, step.v_cache,
               torch.from_numpy(np.ascontiguousarray(tables, dtype=np.int32)).cuda(),
               torch.from_numpy(np.ascontiguousarray(ctx, dtype=np.int32)).cuda(), torch.from_numpy(qs).cuda(),
               step.scale, partition_size=step.partition_size, max_context_len=max_context_len, dev_err=err)
    torch.cuda.synchronize()
    return out, int(err.item())


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: f"h{c[2]}x{c[3]}_d{c[4]}_b{c[5]}_p{c[6]}")
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_prefill_matches_oracle(pa, case, dtype):
    ctx, new, Hq, Hkv, d, B, P = case
    step, q, qs = prefill_inputs(case, dtype)
    out, err = run_prefill(pa, step, q, qs)
    assert err == 0
    ref = oracle.prefill_attention(f64(q), f64(step.k_cache), f64(step.v_cache), step.block_tables,
                                   step.context_lens, qs, step.scale)
    assert_close(f64(out), ref, dtype, torch.float32, str(case))
    # the last new token of each sequence sees its whole context: it is the decode result
    nz = np.array([i for i in range(len(ctx)) if new[i] > 0])
    last = torch.from_numpy(qs[1:][nz] - 1).long().cuda()
    dec = torch.empty(len(nz), Hq, d, dtype=torch.float32, device="cuda")
    pa.decode(dec, q[last].contiguous(), step.k_cache, step.v_cache,
              torch.from_numpy(np.ascontiguousarray(step.block_tables[nz])).cuda(),
              torch.from_numpy(np.ascontiguousarray(step.context_lens[nz])).cuda(), step.scale, partition_size=P)
    torch.cuda.synchronize()
    if pa.prefill_uses_tensor_cores(dtype, Hq, Hkv, d, B):
        # another kernel, another summation order: equal up to both error bounds
        assert float((out[last] - dec).abs().max()) <= 2 * TOL_BF16
    else:
        # the same decode kernels on the same rows: bit for bit
        assert torch.equal(out[last], dec)


def test_prefill_many_sequences_plan_chunks(pa):
    """1500 sequences (the plan kernel walks them 1024 at a time), 1-3 new tokens
    each over short contexts, on the tensor-core path."""
    rng = np.random.default_rng(8)
    S = 1500
    new = rng.integers(1, 4, size=S)
    ctx = new + rng.integers(0, 40, size=S)
    case = (ctx.tolist(), new.tolist(), 8, 2, 64, 16, 32)
    assert pa.prefill_uses_tensor_cores(torch.bfloat16, 8, 2, 64, 16)
    step, q, qs = prefill_inputs(case, torch.bfloat16)
    out, err = run_prefill(pa, step, q, qs)
    assert err == 0
    ref = oracle.prefill_attention(f64(q), f64(step.k_cache), f64(step.v_cache), step.block_tables,
                                   step.context_lens, qs, step.scale)
    assert_close(f64(out), ref, torch.bfloat16, torch.float32, "1500 sequences")


def test_prefill_path_choice(pa):
    bf, f32 = torch.bfloat16, torch.float32
    assert pa.prefill_uses_tensor_cores(bf, 32, 8, 128, 16)
    assert pa.prefill_uses_tensor_cores(bf, 32, 32, 64, 8)
    assert pa.prefill_uses_tensor_cores(bf, 128, 1, 128, 32)     # group 128: one token per tile
    assert not pa.prefill_uses_tensor_cores(f32, 32, 8, 128, 16)
    assert not pa.prefill_uses_tensor_cores(bf, 32, 8, 128, 4)
    assert not pa.prefill_uses_tensor_cores(bf, 12, 4, 128, 16)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["out_f32", "out_bf16"])
def test_prefill_tensor_core_bf16_output(pa, out_dtype):
    case = ([300, 1029, 64, 1], [300, 45, 64, 1], 32, 8, 128, 16, 128)
    step, q, qs = prefill_inputs(case, torch.bfloat16)
    out, err = run_prefill(pa, step, q, qs, out_dtype=out_dtype)
    assert err == 0
    ref = oracle.prefill_attention(f64(q), f64(step.k_cache), f64(step.v_cache), step.block_tables,
                                   step.context_lens, qs, step.scale)
    assert_close(f64(out), ref, torch.bfloat16, out_dtype, "prefill out " + str(out_dtype))


def test_prefill_reservation_and_free_blocks_are_ignored(pa):
    """NaN in every free block and reservation slot: the tensor-core prefill gives
    the same output as without them, bit for bit, and a finite one."""
    case = ([7, 40, 100, 333], [7, 3, 33, 100], 16, 4, 128, 16, 64)
    assert pa.prefill_uses_tensor_cores(torch.bfloat16, 16, 4, 128, 16)
    clean, q, qs = prefill_inputs(case, torch.bfloat16, poison=False)
    dirty, _, _ = prefill_inputs(case, torch.bfloat16, poison=True)
    for st in (clean, dirty):   # the step's own token of each sequence is written first
        pa.reshape_and_cache(st.new_key, st.new_value, st.k_cache, st.v_cache,
                             torch.from_numpy(st.slot_mapping).cuda())
    a, ea = run_prefill(pa, clean, q, qs)
    b, eb = run_prefill(pa, dirty, q, qs)
    assert ea == 0 and eb == 0
    assert torch.isfinite(b).all()
    assert torch.equal(a, b)


@pytest.mark.parametrize("where", ["value", "key"])
def test_prefill_tensor_core_non_finite_visible_value(pa, where):
    """The tensor-core prefill reads a tile's K/V once for all 128 query rows of a
    unit (32 new tokens x 4 heads here), so a NaN value element at a visible
    position t reaches that output column of every row of the unit holding t:
    rows at positions >= t, as in plain attention, and also the unit's earlier
    rows (the documented departure; their weight for t is 0, but 0 * NaN is
    NaN).  A NaN key at t is masked per row before the softmax and reaches only
    rows at positions >= t (all their columns).  Everything else matches the
    oracle; other kv heads are untouched."""
    cached, new, Hq, Hkv, d, B = 40, 100, 32, 8, 128, 16
    case = ([cached + new], [new], Hq, Hkv, d, B, 64)
    assert pa.prefill_uses_tensor_cores(torch.bfloat16, Hq, Hkv, d, B)
    step, q, qs = prefill_inputs(case, torch.bfloat16)
    ref_clean = oracle.prefill_attention(f64(q), f64(step.k_cache), f64(step.v_cache), step.block_tables,
                                         step.context_lens, qs, step.scale)
    t = 80                                     # a position inside the second unit (new tokens 32..63)
    pool = step.v_cache if where == "value" else step.k_cache
    pool[int(step.block_tables[0, t // B]), 0, t % B, 5] = float("nan")   # kv head 0 only
    out, err = run_prefill(pa, step, q, qs)
    assert err == 0
    got = f64(out)
    pos = cached + np.arange(new)
    g = Hq // Hkv
    tq = 128 // g                              # new tokens per unit
    unit_last = np.minimum((np.arange(new) // tq + 1) * tq, new) - 1 + cached
    for h in range(Hq):
        if h >= g:                             # heads of the other kv heads: plain parity
            assert_close(got[:, h], ref_clean[:, h], torch.bfloat16, torch.float32, f"head {h}")
            continue
        late = pos >= t
        if where == "key":
            # a NaN score: the whole row is NaN for every row that sees t, nothing else changes
            assert not np.isfinite(got[late, h]).any(), "rows at or after the NaN key must be NaN"
            clean = ~late
            assert_close(got[clean, h], ref_clean[clean, h], torch.bfloat16, torch.float32, f"head {h}")
            continue
        # a NaN in value column e: column e is NaN for the rows at or after t and for
        # the earlier rows of the unit holding t (0 * NaN inside the tile's P.V);
        # every other element equals plain attention
        e = 5
        reached = (~late) & (unit_last >= t)
        assert reached.sum() > 0
        assert not np.isfinite(got[late, h, e]).any(), "column e of rows at or after t"
        assert not np.isfinite(got[reached, h, e]).any(), "column e of the earlier rows of t's unit"
        rest = ~(late | reached)
        assert rest.sum() > 0
        assert_close(got[rest, h], ref_clean[rest, h], torch.bfloat16, torch.float32, f"head {h} other rows")
        cols = np.arange(d) != e
        assert_close(got[~rest, h][:, cols], ref_clean[~rest, h][:, cols], torch.bfloat16, torch.float32,
                     f"head {h} other columns")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_prefill_more_new_tokens_than_context(pa, dtype):
    """n_s > context_len is flagged; positions below zero see nothing (zeros), the
    others are the causal result over what exists."""
    case = ([40, 50], [10, 20], 8, 2, 64, 16, 32)
    step, q, qs = prefill_inputs(case, dtype)
    ctx = np.array([5, 50], dtype=np.int32)       # sequence 0: 10 new tokens but 5 in the pool
    out, err = run_prefill(pa, step, q, qs, ctx=ctx)
    assert err & pa.DEVERR_CONTEXT
    got = f64(out)
    assert np.all(got[:5] == 0.0)                 # positions -5 .. -1
    ref = oracle.prefill_attention(f64(q[5:]), f64(step.k_cache), f64(step.v_cache), step.block_tables,
                                   ctx, np.array([0, 5, 25], dtype=np.int32), step.scale)
    assert_close(got[5:], ref, dtype, torch.float32, "excess new tokens")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "f32"])
def test_prefill_bad_block_id_is_flagged(pa, dtype):
    case = ([64, 64], [16, 16], 8, 2, 64, 16, 32)
    step, q, qs = prefill_inputs(case, dtype)
    tables = step.block_tables.copy()
    tables[1, 1] = step.num_blocks + 5            # tokens 16..31 of sequence 1 live nowhere
    out, err = run_prefill(pa, step, q, qs, tables=tables)
    assert err & pa.DEVERR_BLOCK_ID
    assert torch.isfinite(out).all()
    ref = oracle.prefill_attention(f64(q[:16]), f64(step.k_cache), f64(step.v_cache), step.block_tables[:1],
                                   step.context_lens[:1], qs[:2], step.scale)
    assert_close(f64(out[:16]), ref, dtype, torch.float32, "sequence with valid blocks")


def test_prefill_chunk_full_size_sampled(pa):
    """The chunked-prefill workload timed by the benchmark (16 sequences x (1024
    cached + 256 new tokens), 32 q / 8 kv heads, d 128, block 16), in the same
    launch configuration; sampled rows against the oracle one by one."""
    step = to_device(W.prefill_chunk())
    T = step.q.shape[0]
    out = torch.empty(T, step.num_heads, step.head_dim, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    qs = step.query_start
    kc, vc = step.k_cache.clone(), step.v_cache.clone()
    pa.reshape_and_cache(step.new_key, step.new_value, kc, vc, torch.from_numpy(step.slot_mapping).cuda(),
                         dev_err=err)
    pa.prefill(out, step.q, kc, vc, torch.from_numpy(step.block_tables).cuda(),
               torch.from_numpy(step.context_lens).cuda(), torch.from_numpy(qs).cuda(), step.scale,
               partition_size=step.partition_size, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rng = np.random.default_rng(3)
    g = step.num_heads // step.num_kv_heads
    for s in rng.choice(step.num_seqs, size=4, replace=False):
        c = int(step.context_lens[s])
        n = int(qs[s + 1] - qs[s])
        blocks = step.block_tables[s][: -(-c // step.block_size)]
        kp = SparsePool.fetch(kc, blocks)
        vp = SparsePool.fetch(vc, blocks)
        for i in sorted(set(rng.integers(0, n, size=5).tolist()) | {0, n - 1}):
            pos = c - n + i
            row = int(qs[s]) + i
            for h in rng.choice(step.num_heads, size=4, replace=False):
                kvh = int(h) // g
                k_rows = oracle.gather_kv(kp, step.block_tables[s], pos + 1, kvh)
                v_rows = oracle.gather_kv(vp, step.block_tables[s], pos + 1, kvh)
                ref = oracle.decode_attention_one(f64(step.q[row, h]), k_rows, v_rows, step.scale)
                assert_close(f64(out[row, h]), ref, torch.bfloat16, torch.bfloat16, f"seq {s} token {i} head {h}")
