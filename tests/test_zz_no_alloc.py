"""pa_decode_noalloc: decode attention for callers that cannot allocate device
memory (a host program whose device memory is planned once at start-up, a
latency-critical caller that must not pay cudaMalloc/cudaFree, a foreign caller
linking only the C ABI).  Its workspace is a fixed array inside the library.

The entry point is called through the C ABI (ctypes, raw pointers) on three
batches in a row (fp32 and bf16 outputs, with and without a context bound), and
each result is compared with pa_decode's on a caller-provided workspace: bit for
bit, and within the tolerances the parity tests use.  Every call after the
first runs over whatever the previous one left in the shared array.
This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


def _abi(pa):
    lib = ctypes.CDLL(pa.LIB_PATH)
    fn = lib.pa_decode_noalloc
    restype, argtypes = pa.SIGNATURES["pa_decode_noalloc"]
    fn.restype, fn.argtypes = restype, argtypes
    return fn


def _call_noalloc(fn, pa, step, tables, ctx, out, err, max_context_len=0):
    kc, vc = step.k_cache, step.v_cache
    NB, Hkv, B, d = kc.shape
    return fn(out.data_ptr(), pa.dtype_code(out.dtype), step.q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
              tables.data_ptr(), ctx.data_ptr(), step.num_seqs, step.num_heads, Hkv, d, B, NB,
              tables.shape[1], max_context_len, float(step.scale), step.partition_size, pa.dtype_code(kc.dtype),
              err.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_decode_twice(pa):
    """Each call gives pa_decode's result on a caller workspace bit for bit (both
    run the same kernels on the same inputs) and within the parity tolerance."""
    from paged_kv_cache_382_b200 import workloads as W

    fn = _abi(pa)
    dev = torch.device("cuda")
    batches = [
        # many partitions per sequence: exercises the partials kept in the array
        (W.independent("noalloc_a", [3000, 17, 1, 0, 1029, 512], dtype=torch.bfloat16, num_heads=32,
                       num_kv_heads=8, head_dim=128, block_size=16, seed=31, device=dev,
                       partition_size=256), torch.float32, 0, 2e-3),
        # fp32 path, fewer partitions: the array still holds the first call's partials
        (W.tiny(block_size=4, device=dev, partition_size=32), torch.float32, 0, 1e-5),
        # bf16 output, and a context bound below what the block tables could address
        (W.independent("noalloc_c", [700, 5, 64, 333], dtype=torch.bfloat16, num_heads=16, num_kv_heads=4,
                       head_dim=64, block_size=8, seed=32, device=dev, partition_size=128),
         torch.bfloat16, 704, 2e-3 + 2.0 ** -8),
    ]
    for step, out_dtype, max_ctx, tol in batches:
        tables = torch.from_numpy(step.block_tables.astype(np.int32)).to(dev)
        if max_ctx:
            # room for more blocks than the bound allows, so the bound decides the partials
            pad = torch.full((step.num_seqs, 200), -1, dtype=torch.int32, device=dev)
            tables = torch.cat([tables, pad], dim=1).contiguous()
        ctx = torch.from_numpy(step.context_lens.astype(np.int32)).to(dev)
        shape = (step.num_seqs, step.num_heads, step.head_dim)
        ref = torch.empty(shape, dtype=out_dtype, device=dev)
        got = torch.full(shape, float("nan"), dtype=out_dtype, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        pa.decode(ref, step.q, step.k_cache, step.v_cache, tables, ctx, step.scale, max_context_len=max_ctx,
                  partition_size=step.partition_size, dev_err=err)
        rc = _call_noalloc(fn, pa, step, tables, ctx, got, err, max_context_len=max_ctx)
        assert rc == pa.PA_OK, pa.lib.pa_status_string(rc)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.isfinite(got).all()
        assert torch.equal(got, ref)
        assert float((got.float() - ref.float()).abs().max()) <= tol


def test_noalloc_rejects_batches_beyond_its_array(pa):
    fn = _abi(pa)
    dev = torch.device("cuda")
    # 64 sequences x 64 heads x 256 partitions of partials is far beyond 64 MiB
    S, H, Hkv, d, B, NB, P = 64, 64, 8, 128, 16, 8, 512
    max_blocks = 131072 // B
    need = pa.lib.pa_decode_workspace_bytes(S, H, d, max_blocks * B, P)
    assert need > pa.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(S, H, d, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(NB, Hkv, B, d, dtype=torch.bfloat16, device=dev)
    tables = torch.zeros(S, max_blocks, dtype=torch.int32, device=dev)
    ctx = torch.zeros(S, dtype=torch.int32, device=dev)
    out = torch.zeros(S, H, d, dtype=torch.float32, device=dev)
    rc = fn(out.data_ptr(), pa.PA_F32, q.data_ptr(), kc.data_ptr(), kc.data_ptr(), tables.data_ptr(),
            ctx.data_ptr(), S, H, Hkv, d, B, NB, max_blocks, 0, 0.1, P, pa.PA_BF16, None,
            torch.cuda.current_stream().cuda_stream)
    assert rc == pa.PA_ERR_WORKSPACE
