"""CPU checks of the C ABI: libpa.so loads, exports every function include/pa.h
declares, and rejects bad arguments on the host before any CUDA call."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_382_b200 import build

    build.build()
    from paged_kv_cache_382_b200 import pa as binding

    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*PA_API\s+[\w\s\*]*?\b(pa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ["pa_reshape_and_cache", "pa_decode", "pa_decode_phases", "pa_decode_workspace_bytes",
                     "pa_copy_blocks", "pa_status_string", "pa_version"]:
        assert required in names


def test_library_exports_every_declared_symbol(pa):
    lib = ctypes.CDLL(pa.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(declared_functions()) <= set(pa.SIGNATURES)


def test_library_exports_only_the_c_abi(pa):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split() and line.split()[-2] in "TWVuBD"}
    assert exported == set(declared_functions()), sorted(exported ^ set(declared_functions()))


def test_noalloc_limit_matches_the_header(pa):
    """The binding's copy of PA_NOALLOC_SCRATCH_BYTES is the header's value."""
    text = open(HEADER).read()
    m = re.search(r"#define\s+PA_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "PA_NOALLOC_SCRATCH_BYTES not found in include/pa.h"
    expr = re.sub(r"(\d+)[uUlL]+", r"\1", m.group(1))
    assert re.fullmatch(r"[\d\s\*\+]+", expr), expr
    assert eval(expr) == pa.NOALLOC_SCRATCH_BYTES


def test_status_codes_match_the_header(pa):
    text = open(HEADER).read()
    for name in ["PA_OK", "PA_ERR_INVALID_ARG", "PA_ERR_UNSUPPORTED", "PA_ERR_WORKSPACE", "PA_ERR_CUDA",
                 "PA_ERR_DEVICE_INDEX"]:
        m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
        assert m, name
        assert int(m.group(1)) == getattr(pa, name), name
        assert name.encode() in pa.lib.pa_status_string(int(m.group(1)))


def test_status_strings_and_version(pa):
    assert pa.lib.pa_status_string(0).decode() == "PA_OK"
    assert b"workspace" in pa.lib.pa_status_string(3)
    assert pa.lib.pa_version() >= 100


def test_decode_step_host_validation(pa):
    """pa_decode_step refuses bad scatter, copy or decode arguments before any
    launch (no GPU needed)."""
    f = pa.lib.pa_decode_step
    base = dict(out=256, od=pa.PA_F32, q=256, key=256, value=256, k=256, v=256, slots=256, T=4, pairs=None,
                npairs=0, tables=256, ctx=256, S=4, Hq=32, Hkv=8, d=128, B=16, NB=64, mb=8, maxc=0, scale=0.1,
                P=512, ws=None, wsb=0, dt=pa.PA_BF16, err=None, st=None)

    def call(**over):
        a = {**base, **over}
        return f(a["out"], a["od"], a["q"], a["key"], a["value"], a["k"], a["v"], a["slots"], a["T"], a["pairs"],
                 a["npairs"], a["tables"], a["ctx"], a["S"], a["Hq"], a["Hkv"], a["d"], a["B"], a["NB"], a["mb"],
                 a["maxc"], a["scale"], a["P"], a["ws"], a["wsb"], a["dt"], a["err"], a["st"])

    assert call(key=None) == pa.PA_ERR_INVALID_ARG              # new tokens without keys
    assert call(slots=258) == pa.PA_ERR_INVALID_ARG             # misaligned slot mapping
    assert call(npairs=2) == pa.PA_ERR_INVALID_ARG              # pairs announced, none given
    assert call(T=-1) == pa.PA_ERR_INVALID_ARG
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED                  # the decode's own checks
    assert call(ws=None, wsb=0) == pa.PA_ERR_INVALID_ARG        # no workspace


def test_selftest_host_validation(pa):
    """Bad arguments of the bounded-wait self-test are refused before any launch."""
    f = pa.lib.pa_selftest_bounded_wait
    assert f(None, 1000, None) == pa.PA_ERR_INVALID_ARG              # no error word
    assert f(256, 0, None) == pa.PA_ERR_INVALID_ARG                  # no limit
    assert f(256, 2_000_000_000, None) == pa.PA_ERR_INVALID_ARG      # limit above 1 s
    assert f(258, 1000, None) == pa.PA_ERR_INVALID_ARG               # misaligned error word


def test_workspace_bytes(pa):
    ws = pa.lib.pa_decode_workspace_bytes
    r = lambda n: (n + 255) // 256 * 256  # noqa: E731
    W, cap_max = 3, 256                    # warps (streams, column groups) and split units

    def expect(S, H, D, cap, P):
        parts = max(1, -(-cap // P))
        split = min(cap_max, (S // 2) * parts * H)
        state = (4 * (D // 16) + 4) * 32 * 4
        # header; work list (two int32 pairs per item: code, context, split slot, spare),
        # room for the extra stream items of split shared items; (max, sum) and fp32 partials
        # when a context spans partitions; split units' stream states and their counters
        n = 256 + r((S * parts + (W - 1) * split) * 16)
        if parts > 1:
            n += r(S * H * parts * 8) + r(S * H * parts * D * 4)
        return n + r(split * W * W * state) + r(split * 4)

    assert ws(64, 32, 128, 512, 512) == expect(64, 32, 128, 512, 512)
    assert ws(8, 64, 128, 131072, 512) == expect(8, 64, 128, 131072, 512)
    assert ws(1, 8, 64, 100, 32) == expect(1, 8, 64, 100, 32)       # one sequence: nothing to split
    assert ws(1, 8, 64, 100, 32) == 256 + r(1 * 4 * 16) + r(8 * 4 * 8) + r(8 * 4 * 64 * 4)
    assert ws(-1, 1, 64, 10, 512) == 0
    assert ws(1, 1, 64, 10, 0) == 0


def _decode_call(pa, **over):
    args = dict(out=1 << 20, out_dtype=0, q=1 << 20, k=1 << 20, v=1 << 20, tables=1 << 20, ctx=1 << 20,
                S=4, Hq=4, Hkv=4, D=64, B=16, NB=64, max_blocks=8, max_ctx=0, scale=0.125, P=512,
                ws=1 << 20, ws_bytes=1 << 30, dtype=0, err=None, stream=None, phases=7)
    args.update(over)
    return pa.lib.pa_decode_phases(args["out"], args["out_dtype"], args["q"], args["k"], args["v"],
                                   args["tables"], args["ctx"], args["S"], args["Hq"], args["Hkv"],
                                   args["D"], args["B"], args["NB"], args["max_blocks"], args["max_ctx"],
                                   args["scale"], args["P"], args["ws"], args["ws_bytes"], args["dtype"],
                                   args["err"], args["stream"], args["phases"])


@pytest.mark.parametrize("over,status", [
    (dict(Hq=6, Hkv=4), 1),            # heads not a multiple of kv heads
    (dict(D=96), 2),                   # head_dim
    (dict(B=64), 2),                   # block_size
    (dict(P=48), 2),                   # partition not a multiple of 32
    (dict(P=16384), 2),                # partition too large
    (dict(B=32, P=32 + 32 * 0), 0),    # fine shapes, but S=0 below
    (dict(dtype=5), 1),                # dtype
    (dict(out_dtype=1, dtype=0), 2),   # bf16 output from fp32 input
    (dict(ws=None), 1),                # no workspace
    (dict(ws=(1 << 20) + 8), 1),       # misaligned workspace
    (dict(ws_bytes=10), 3),            # short workspace
    (dict(q=(1 << 20) + 2), 1),        # misaligned q
    (dict(tables=None), 1),
    (dict(scale=float("nan")), 1),
    (dict(phases=0), 1),
    (dict(phases=8), 1),
    (dict(max_ctx=-1), 1),
])
def test_decode_host_validation(pa, over, status):
    if status == 0:
        over = dict(over, S=0)          # an empty batch is a no-op that touches nothing
    assert _decode_call(pa, **over) == status


def test_cache_ops_host_validation(pa):
    L = pa.lib
    assert L.pa_reshape_and_cache(None, None, None, None, None, 0, 8, 128, 16, 64, 1, None, None) == 0
    assert L.pa_reshape_and_cache(None, None, None, None, None, 3, 8, 128, 16, 64, 1, None, None) == 1
    assert L.pa_reshape_and_cache(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 3, 8, 80, 16, 64, 1, None,
                                  None) == 2
    assert L.pa_reshape_and_cache(1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20, 3, 8, 128, 12, 64, 1, None,
                                  None) == 2
    assert L.pa_copy_blocks(None, None, None, 0, 4096, 64, None, None) == 0
    assert L.pa_copy_blocks(None, None, None, 2, 4096, 64, None, None) == 1
    assert L.pa_copy_blocks(1 << 20, 1 << 20, 1 << 20, 2, 4095, 64, None, None) == 1


def test_binding_marshals_no_cpu_tensors(pa):
    import torch

    k = torch.zeros(4, 2, 16, 64)
    with pytest.raises(ValueError, match="CUDA"):
        pa.reshape_and_cache(torch.zeros(1, 2, 64), torch.zeros(1, 2, 64), k, k.clone(),
                             torch.zeros(1, dtype=torch.int64))
