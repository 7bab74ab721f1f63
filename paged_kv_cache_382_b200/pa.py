"""ctypes binding of libpa.so: argument marshalling only.

Every function checks the torch tensors it is given (device, dtype,
contiguity), passes raw device pointers and the current CUDA stream to the C
ABI declared in ``include/pa.h``, and raises ``PagedAttentionError`` on a
non-zero status.  All arithmetic happens in the library's CUDA kernels; there
is no CPU fallback -- importing this module raises ImportError when libpa.so
has not been built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

PA_F32, PA_BF16 = 0, 1
PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_CUDA, PA_ERR_DEVICE_INDEX = 0, 1, 2, 3, 4, 5
DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_CONTEXT, DEVERR_COPY, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
PHASE_PLAN, PHASE_ATTEND, PHASE_REDUCE, PHASE_ALL = 0x1, 0x2, 0x4, 0x7

_vp, _i, _i32p, _i64p, _sz, _f = (ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.c_size_t, ctypes.c_float)

_DECODE_ARGS = [_vp, _i, _vp, _vp, _vp, _i32p, _i32p, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                _vp, _sz, _i, _i32p, _vp]

SIGNATURES = {
    "pa_reshape_and_cache": (_i, [_vp, _vp, _vp, _vp, _i64p, _i, _i, _i, _i, _i, _i, _i32p, _vp]),
    "pa_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "pa_decode": (_i, _DECODE_ARGS),
    "pa_decode_phases": (_i, _DECODE_ARGS + [_i]),
    "pa_decode_step": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _i64p, _i, _i64p, _i, _i32p, _i32p, _i, _i, _i, _i,
                            _i, _i, _i, _i, _f, _i, _vp, _sz, _i, _i32p, _vp]),
    "pa_copy_blocks": (_i, [_vp, _vp, _i64p, _i, _sz, _i, _i32p, _vp]),
    "pa_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "pa_prefill_uses_tensor_cores": (_i, [_i, _i, _i, _i, _i]),
    "pa_prefill": (_i, [_vp, _i, _vp, _vp, _vp, _i32p, _i32p, _i32p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                        _i, _vp, _sz, _i, _i32p, _vp]),
    "pa_decode_noalloc": (_i, [_vp, _i, _vp, _vp, _vp, _i32p, _i32p, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                               _i, _i, _i32p, _vp]),
    "pa_bm_create": (ctypes.c_void_p, [_i, _i, _vp, _i]),
    "pa_bm_destroy": (None, [_vp]),
    "pa_bm_add_sequence": (_i, [_vp, ctypes.c_int64]),
    "pa_bm_fork": (_i, [_vp, ctypes.c_int64, ctypes.c_int64]),
    "pa_bm_free": (_i, [_vp, ctypes.c_int64]),
    "pa_bm_append": (_i, [_vp, ctypes.c_int64, _vp, _i, _vp, _vp, _i, ctypes.POINTER(ctypes.c_int),
                          ctypes.POINTER(ctypes.c_int)]),
    "pa_bm_append_batch": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _i, ctypes.POINTER(ctypes.c_int),
                                ctypes.POINTER(ctypes.c_int)]),
    "pa_bm_block_table": (_i, [_vp, ctypes.c_int64, _vp, _i, ctypes.POINTER(ctypes.c_int),
                               ctypes.POINTER(ctypes.c_int64)]),
    "pa_bm_num_free": (_i, [_vp]),
    "pa_bm_ref_count": (_i, [_vp, _i]),
    "pa_selftest_bounded_wait": (_i, [_i32p, ctypes.c_uint64, _vp]),
    "pa_status_string": (ctypes.c_char_p, [_i]),
    "pa_version": (_i, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built: run `python -m paged_kv_cache_382_b200.build` "
            "(needs nvcc); this package has no CPU fallback")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (restype, argtypes) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = restype
        fn.argtypes = argtypes
    return lib


lib = _load()


class PagedAttentionError(RuntimeError):
    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {lib.pa_status_string(status).decode()}")
        self.status = status


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PagedAttentionError(what, status)


def dtype_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return PA_F32
    if dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"unsupported dtype {dtype}; the kernels take float32 or bfloat16")


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _opt_err(dev_err: Optional[torch.Tensor]) -> Optional[int]:
    if dev_err is None:
        return None
    return _dev(dev_err, "dev_err", torch.int32)


def reshape_and_cache(key: torch.Tensor, value: torch.Tensor, k_cache: torch.Tensor,
                      v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                      dev_err: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    """Write key/value [T][Hkv][d] into the pools [NB][Hkv][B][d] at slot_mapping (int64 [T])."""
    NB, Hkv, B, d = k_cache.shape
    if tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must have the same shape")
    T = key.shape[0]
    if tuple(key.shape) != (T, Hkv, d) or tuple(value.shape) != (T, Hkv, d):
        raise ValueError("key/value must be [num_tokens][num_kv_heads][head_dim]")
    if tuple(slot_mapping.shape) != (T,):
        raise ValueError("slot_mapping must be [num_tokens]")
    dt = k_cache.dtype
    rc = lib.pa_reshape_and_cache(
        _dev(key, "key", dt), _dev(value, "value", dt), _dev(k_cache, "k_cache", dt),
        _dev(v_cache, "v_cache", dt), _dev(slot_mapping, "slot_mapping", torch.int64), T, Hkv, d, B,
        NB, dtype_code(dt), _opt_err(dev_err), _stream_handle(stream))
    _check(rc, "pa_reshape_and_cache")


def decode_workspace_bytes(num_seqs: int, num_heads: int, head_dim: int, max_context_len: int,
                           partition_size: int = 512) -> int:
    n = lib.pa_decode_workspace_bytes(num_seqs, num_heads, head_dim, max_context_len, partition_size)
    if n == 0:
        raise ValueError("invalid arguments for pa_decode_workspace_bytes")
    return int(n)


def decode_capacity(block_tables: torch.Tensor, block_size: int, max_context_len: int = 0) -> int:
    """The context bound the library uses: max_context_len, or max_blocks * block_size if 0."""
    cap = block_tables.shape[1] * block_size
    return cap if max_context_len <= 0 else min(cap, max_context_len)


def alloc_workspace(num_seqs: int, num_heads: int, head_dim: int, capacity: int,
                    partition_size: int = 512, device=None) -> torch.Tensor:
    n = decode_workspace_bytes(num_seqs, num_heads, head_dim, capacity, partition_size)
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda"))


def decode(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
           block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, *,
           max_context_len: int = 0, partition_size: int = 512,
           workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None, phases: int = PHASE_ALL) -> torch.Tensor:
    """Paged decode attention; writes and returns ``out`` [S][Hq][d]."""
    NB, Hkv, B, d = k_cache.shape
    S, Hq, dq = q.shape
    if dq != d or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q, k_cache and v_cache disagree on head_dim / shape")
    if tuple(out.shape) != (S, Hq, d):
        raise ValueError("out must be [num_seqs][num_heads][head_dim]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs][max_blocks] and context_lens [num_seqs]")
    dt = k_cache.dtype
    if workspace is None:
        cap = decode_capacity(block_tables, B, max_context_len)
        workspace = alloc_workspace(S, Hq, d, cap, partition_size, q.device)
    rc = lib.pa_decode_phases(
        _dev(out, "out"), dtype_code(out.dtype), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt),
        _dev(v_cache, "v_cache", dt), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), S, Hq, Hkv, d, B, NB,
        block_tables.shape[1], max_context_len, float(scale), partition_size,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), dtype_code(dt),
        _opt_err(dev_err), _stream_handle(stream), phases)
    _check(rc, "pa_decode")
    return out


def decode_step(out: torch.Tensor, q: torch.Tensor, key: torch.Tensor, value: torch.Tensor,
                k_cache: torch.Tensor, v_cache: torch.Tensor, slot_mapping: torch.Tensor,
                block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, *,
                copy_pairs: Optional[torch.Tensor] = None, max_context_len: int = 0, partition_size: int = 512,
                workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """One decode step in one call: copy-on-write copies (int64 [n][2]), the
    scatter of key/value [T][Hkv][d] through slot_mapping, and paged decode
    attention; writes and returns ``out`` [S][Hq][d]."""
    NB, Hkv, B, d = k_cache.shape
    S, Hq, dq = q.shape
    T = key.shape[0]
    if dq != d or tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != (S, Hq, d):
        raise ValueError("q / out must be [num_seqs][num_heads][head_dim] over the pool's head_dim")
    if tuple(key.shape) != (T, Hkv, d) or tuple(value.shape) != (T, Hkv, d) or tuple(slot_mapping.shape) != (T,):
        raise ValueError("key/value must be [T][num_kv_heads][head_dim] and slot_mapping [T]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or tuple(context_lens.shape) != (S,):
        raise ValueError("block_tables must be [num_seqs][max_blocks] and context_lens [num_seqs]")
    npairs = 0 if copy_pairs is None else int(copy_pairs.shape[0])
    if npairs and (copy_pairs.dim() != 2 or copy_pairs.shape[1] != 2):
        raise ValueError("copy_pairs must be int64 [n][2]")
    dt = k_cache.dtype
    if workspace is None:
        cap = decode_capacity(block_tables, B, max_context_len)
        workspace = alloc_workspace(S, Hq, d, cap, partition_size, q.device)
    rc = lib.pa_decode_step(
        _dev(out, "out"), dtype_code(out.dtype), _dev(q, "q", dt), _dev(key, "key", dt) if T else None,
        _dev(value, "value", dt) if T else None, _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        _dev(slot_mapping, "slot_mapping", torch.int64) if T else None, T,
        _dev(copy_pairs, "copy_pairs", torch.int64) if npairs else None, npairs,
        _dev(block_tables, "block_tables", torch.int32), _dev(context_lens, "context_lens", torch.int32), S, Hq,
        Hkv, d, B, NB, block_tables.shape[1], max_context_len, float(scale), partition_size,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), dtype_code(dt), _opt_err(dev_err),
        _stream_handle(stream))
    _check(rc, "pa_decode_step")
    return out


def prefill(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
            block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor, scale: float,
            *, max_context_len: int = 0, partition_size: int = 512,
            workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Causal attention of new tokens q [T][Hq][d] (sequence s owns rows
    query_start[s]..query_start[s+1]-1) against the paged context; writes ``out``."""
    NB, Hkv, B, d = k_cache.shape
    T, Hq, dq = q.shape
    S = context_lens.shape[0]
    if dq != d or tuple(out.shape) != (T, Hq, d) or tuple(query_start.shape) != (S + 1,):
        raise ValueError("q/out must be [num_tokens][num_heads][head_dim], query_start [num_seqs + 1]")
    if block_tables.dim() != 2 or block_tables.shape[0] != S:
        raise ValueError("block_tables must be [num_seqs][max_blocks]")
    dt = k_cache.dtype
    if workspace is None:
        cap = decode_capacity(block_tables, B, max_context_len)
        n = lib.pa_prefill_workspace_bytes(T, Hq, d, cap, partition_size)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    rc = lib.pa_prefill(
        _dev(out, "out"), dtype_code(out.dtype), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt),
        _dev(v_cache, "v_cache", dt), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), _dev(query_start, "query_start", torch.int32), S, T,
        Hq, Hkv, d, B, NB, block_tables.shape[1], max_context_len, float(scale), partition_size,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), dtype_code(dt), _opt_err(dev_err),
        _stream_handle(stream))
    _check(rc, "pa_prefill")
    return out


def prefill_uses_tensor_cores(dtype: torch.dtype, num_heads: int, num_kv_heads: int, head_dim: int,
                              block_size: int) -> bool:
    """Whether ``prefill`` serves this shape with the tensor-core (tcgen05) kernel."""
    return bool(lib.pa_prefill_uses_tensor_cores(dtype_code(dtype), num_heads, num_kv_heads, head_dim,
                                                 block_size))


def selftest_bounded_wait(dev_err: torch.Tensor, limit_ns: int = 1_000_000,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    """Launch the device self-test of the bounded wait: it must OR
    DEVERR_TIMEOUT into dev_err after limit_ns and return."""
    rc = lib.pa_selftest_bounded_wait(_dev(dev_err, "dev_err", torch.int32), int(limit_ns), _stream_handle(stream))
    _check(rc, "pa_selftest_bounded_wait")


def copy_blocks(k_cache: torch.Tensor, v_cache: torch.Tensor, src_dst_pairs: torch.Tensor,
                dev_err: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """Copy whole blocks src -> dst (int64 [n][2] on the device) in both pools."""
    if tuple(v_cache.shape) != tuple(k_cache.shape) or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache must match")
    n = src_dst_pairs.shape[0]
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [num_pairs][2]")
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    rc = lib.pa_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                            _dev(src_dst_pairs, "src_dst_pairs", torch.int64), n, block_bytes,
                            k_cache.shape[0], _opt_err(dev_err), _stream_handle(stream))
    _check(rc, "pa_copy_blocks")


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def decode_noalloc(out: torch.Tensor, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                   block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float, *,
                   max_context_len: int = 0, partition_size: int = 512,
                   dev_err: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Paged decode attention for callers that cannot allocate device memory: like
    ``decode`` but with the workspace in a fixed 64 MiB array inside the library
    (shared by all calls on a device; calls that overlap on the GPU race)."""
    NB, Hkv, B, d = k_cache.shape
    S, Hq, _ = q.shape
    dt = k_cache.dtype
    rc = lib.pa_decode_noalloc(
        _dev(out, "out"), dtype_code(out.dtype), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt),
        _dev(v_cache, "v_cache", dt), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), S, Hq, Hkv, d, B, NB, block_tables.shape[1],
        max_context_len, float(scale), partition_size, dtype_code(dt), _opt_err(dev_err),
        _stream_handle(stream))
    _check(rc, "pa_decode_noalloc")
    return out


class NativeBlockManager:
    """Handle on the library's host block manager (``pa_bm_*``): free list, ref
    counts, lazy allocation, fork, copy-on-write planning and, optionally,
    prefix caching by chained block keys.  Host memory only."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None, prefix_cache: bool = False):
        import numpy as np

        self._np = np
        self.block_size = int(block_size)
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            order = self._order.ctypes.data
        self._h = lib.pa_bm_create(int(num_blocks), int(block_size), order, int(bool(prefix_cache)))
        if not self._h:
            raise ValueError("pa_bm_create rejected its arguments")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib.pa_bm_destroy(h)
            self._h = None

    def add(self, seq_id: int) -> None:
        _check(lib.pa_bm_add_sequence(self._h, seq_id), "pa_bm_add_sequence")

    def fork(self, parent: int, child: int) -> None:
        _check(lib.pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def free(self, seq_id: int) -> None:
        _check(lib.pa_bm_free(self._h, seq_id), "pa_bm_free")

    def append(self, seq_id: int, tokens):
        """Append tokens (a count, or token ids when prefix caching).  Returns
        (slots int64 array, [(src, dst) copies], tokens served from the cache)."""
        np = self._np
        ids = None
        if isinstance(tokens, int):
            n = tokens
        else:
            ids = np.ascontiguousarray(tokens, dtype=np.int32)
            n = len(ids)
        slots = np.empty(max(n, 1), dtype=np.int64)
        cap = max(n, 1)
        copies = np.empty(2 * cap, dtype=np.int64)
        ncopies, ncached = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib.pa_bm_append(self._h, seq_id, None if ids is None else ids.ctypes.data, n, slots.ctypes.data,
                              copies.ctypes.data, cap, ctypes.byref(ncopies), ctypes.byref(ncached))
        _check(rc, "pa_bm_append")
        pairs = [(int(copies[2 * i]), int(copies[2 * i + 1])) for i in range(ncopies.value)]
        return slots[:n], pairs, ncached.value

    def append_batch(self, seq_ids, tokens, max_copies=None, counts=None):
        """One call for a batch: tokens[k] (a count, or token ids when prefix
        caching) appended to seq_ids[k].  With `counts` given, `tokens` is
        instead one flat array of all the token ids in order (or None without
        prefix caching), as a serving loop holds them.  Returns (slots of all
        new tokens in order, [(src, dst) copies], tokens served from the cache)."""
        np = self._np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        if counts is not None:
            counts = np.ascontiguousarray(counts, dtype=np.int32)
            toks = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
            if toks is not None and toks.size != int(counts.sum()):
                raise ValueError("tokens must hold sum(counts) token ids")
        elif all(isinstance(t, (int, np.integer)) for t in tokens):
            counts = np.ascontiguousarray(tokens, dtype=np.int32)
            toks = None
        else:
            counts = np.array([len(t) for t in tokens], dtype=np.int32)
            toks = np.ascontiguousarray(np.concatenate([np.asarray(t, dtype=np.int32) for t in tokens])
                                        if len(tokens) else np.zeros(0, dtype=np.int32), dtype=np.int32)
        total = int(counts.sum())
        slots = np.empty(max(total, 1), dtype=np.int64)
        cap = max(total, 1) if max_copies is None else int(max_copies)
        copies = np.empty(2 * max(cap, 1), dtype=np.int64)
        ncopies, ncached = ctypes.c_int(0), ctypes.c_int(0)
        rc = lib.pa_bm_append_batch(self._h, len(ids), ids.ctypes.data, counts.ctypes.data,
                                    None if toks is None else toks.ctypes.data, slots.ctypes.data,
                                    copies.ctypes.data, cap, ctypes.byref(ncopies), ctypes.byref(ncached))
        _check(rc, "pa_bm_append_batch")
        pairs = [(int(copies[2 * i]), int(copies[2 * i + 1])) for i in range(ncopies.value)]
        return slots[:total], pairs, ncached.value

    def block_table(self, seq_id: int):
        np = self._np
        nb, nt = ctypes.c_int(0), ctypes.c_int64(0)
        rc = lib.pa_bm_block_table(self._h, seq_id, None, 0, ctypes.byref(nb), ctypes.byref(nt))
        if rc not in (PA_OK, PA_ERR_WORKSPACE):
            _check(rc, "pa_bm_block_table")
        out = np.empty(max(nb.value, 1), dtype=np.int32)
        _check(lib.pa_bm_block_table(self._h, seq_id, out.ctypes.data, len(out), ctypes.byref(nb),
                                     ctypes.byref(nt)), "pa_bm_block_table")
        return [int(b) for b in out[: nb.value]]

    def num_tokens(self, seq_id: int) -> int:
        nb, nt = ctypes.c_int(0), ctypes.c_int64(0)
        lib.pa_bm_block_table(self._h, seq_id, None, 0, ctypes.byref(nb), ctypes.byref(nt))
        return int(nt.value)

    @property
    def num_free(self) -> int:
        return int(lib.pa_bm_num_free(self._h))

    def ref_count(self, block: int) -> int:
        return int(lib.pa_bm_ref_count(self._h, block))
