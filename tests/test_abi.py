"""The C-ABI library loads, exports every entry point include/dma.h declares,
and validates arguments on the host before launching anything.  No test here
touches a GPU: every call below is rejected by host-side checks."""
import ctypes
import os
import re

import pytest

import trainable_dynamic_mask_b200 as dma
from trainable_dynamic_mask_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dma.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    if not os.path.exists(_lib.LIB_PATH):
        from trainable_dynamic_mask_b200 import build
        build.build()
    return dma.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dma_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound():
    names = declared_functions()
    assert len(names) >= 11
    lib = dma.load()
    for n in names:
        assert hasattr(lib, n), f"{n} missing from libdma.so"
    assert sorted(_lib.exported_names()) == names


def test_abi_version_and_status_strings():
    assert dma.abi_version() == 2
    lib = dma.load()
    for code in range(6):
        s = lib.dma_status_string(code).decode()
        assert s.startswith(_lib.STATUS_NAMES[code])
    assert lib.dma_status_string(99).decode() == "DMA_ERR_UNKNOWN"


def _ws_size(p):
    n = ctypes.c_size_t(0)
    st = dma.load().dma_workspace_size(ctypes.byref(p), ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize("kw,expect", [
    (dict(B=1, H=2, Hkv=1, N=256, d=64, w=64), OK),
    (dict(B=1, H=3, Hkv=2, N=256, d=64, w=64), INVALID),        # H % Hkv
    (dict(B=1, H=2, Hkv=1, N=256, d=96, w=64), UNSUPPORTED),    # head dim
    (dict(B=1, H=2, Hkv=1, N=256, d=64, w=0), INVALID),         # window
    (dict(B=0, H=2, Hkv=1, N=256, d=64, w=4), INVALID),
    (dict(B=1, H=2, Hkv=1, N=16385, d=64, w=4), UNSUPPORTED),   # prefill row limit
    (dict(B=1, H=2, Hkv=1, N=16384, d=128, w=4), OK),
    (dict(B=1, H=2, Hkv=1, N=65536, d=128, w=4, Nq=1), OK),     # decode has no such limit
    (dict(B=1, H=2, Hkv=1, N=256, d=64, w=4, Nq=7), OK),        # a chunk of 7 queries at positions 249..255
    (dict(B=1, H=2, Hkv=1, N=256, d=64, w=4, Nq=257), INVALID), # more queries than keys
    (dict(B=300, H=256, Hkv=1, N=256, d=64, w=4), UNSUPPORTED), # grid limit on B*H
])
def test_params_validation(kw, expect):
    p = dma.make_params(**kw)
    st, _ = _ws_size(p)
    assert st == expect


def test_misaligned_head_windows_pointer():
    p = dma.make_params(1, 2, 1, 256, 64, 64, w_heads=(1 << 20) + 4)
    assert _ws_size(p)[0] == INVALID
    p = dma.make_params(1, 2, 1, 256, 64, 64, w_heads=1 << 20)
    assert _ws_size(p)[0] == OK


def test_decode_selection_stride_with_head_windows():
    # without per-head windows the rows hold min(w, N) keys; with them the stride is w whatever N is
    assert dma.workspace_layout(dma.make_params(1, 2, 1, 100, 64, 300, Nq=1)).sel_len == 100
    assert dma.workspace_layout(dma.make_params(1, 2, 1, 100, 64, 300, Nq=1, w_heads=1 << 20)).sel_len == 300


def test_flags():
    p = dma.make_params(1, 2, 1, 256, 64, 64)
    p.flags = 2
    assert _ws_size(p)[0] == INVALID
    # a forward-only problem keeps nothing for a backward: a smaller workspace
    full = dma.workspace_size(dma.make_params(1, 16, 8, 4096, 128, 1024))
    fwd = dma.workspace_size(dma.make_params(1, 16, 8, 4096, 128, 1024, forward_only=True))
    assert full - fwd >= 16 * 4096 * 128 * 2


def test_bad_dtype_and_scale():
    p = dma.make_params(1, 2, 1, 256, 64, 64)
    p.dtype = 7
    assert _ws_size(p)[0] == INVALID
    p = dma.make_params(1, 2, 1, 256, 64, 64, scale=float("nan"))
    assert _ws_size(p)[0] == INVALID


def test_workspace_layout_plan():
    p = dma.make_params(B=1, H=16, Hkv=8, N=4096, d=128, w=1024)
    lay = dma.workspace_layout(p)
    assert lay.n_blocks == 32
    assert lay.list_cap == 1024 + 128
    assert lay.sel_len == 0
    for off in (lay.off_status, lay.off_counts, lay.off_lists):
        assert off % 256 == 0
    assert lay.off_counts >= lay.off_status + 4
    assert lay.off_lists >= lay.off_counts + 16 * 32 * 2 * 4
    assert lay.bytes >= lay.off_lists + 16 * 32 * lay.list_cap * 4
    assert dma.workspace_size(p) == lay.bytes
    # window wider than the sequence: lists never exceed the padded sequence
    lay2 = dma.workspace_layout(dma.make_params(B=1, H=1, Hkv=1, N=300, d=64, w=5000))
    assert lay2.list_cap == 384 and lay2.n_blocks == 3
    # decode: selection region
    lay3 = dma.workspace_layout(dma.make_params(B=8, H=32, Hkv=8, N=65536, d=128, w=2048, Nq=1))
    assert lay3.sel_len == 2048 and lay3.n_blocks == 0 and lay3.off_sel % 256 == 0


# The fake-pointer checks run in a child process that sees no GPU, so a call
# that wrongly passed validation could never launch a kernel on real memory.
_FAKE_CHECKS = r"""
import ctypes, sys
sys.path.insert(0, %(root)r)
import trainable_dynamic_mask_b200 as dma
OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
FAKE = 1 << 20   # 16-byte aligned, non-null, never dereferenced on the host
lib = dma.load()
def need_of(p):
    n = ctypes.c_size_t(0)
    assert lib.dma_workspace_size(ctypes.byref(p), ctypes.byref(n)) == OK
    return n.value
p = dma.make_params(1, 2, 1, 256, 64, 64)
pp = ctypes.byref(p)
need = need_of(p)
assert lib.dma_gate(pp, None, FAKE, FAKE, FAKE, None, None, 0, None) == INVALID
assert lib.dma_gate(pp, FAKE + 4, FAKE, FAKE, FAKE, None, None, 0, None) == INVALID
assert lib.dma_gate(pp, FAKE, FAKE, FAKE, FAKE, FAKE + 8, None, 0, None) == INVALID
assert lib.dma_topk_mask(pp, FAKE, FAKE, None, need, None) == WORKSPACE
assert lib.dma_topk_mask(pp, FAKE, FAKE, FAKE, need - 1, None) == WORKSPACE
assert lib.dma_topk_mask(pp, FAKE, FAKE, FAKE + 4, need, None) == WORKSPACE
assert lib.dma_topk_mask(pp, FAKE, None, FAKE, need, None) == INVALID
pd = dma.make_params(1, 2, 1, 256, 64, 64, Nq=1)
needd = need_of(pd)
assert lib.dma_topk_mask(ctypes.byref(pd), FAKE, FAKE, FAKE, needd, None) == INVALID
assert lib.dma_attn_fwd(pp, FAKE, FAKE, FAKE, FAKE, None, FAKE, need, FAKE, FAKE, None) == INVALID
# attn_bwd(p, Q, K, V, delta, evict, ws, ws_bytes, O, LSE, dO, dQ, dK, dV, d_delta, stream)
args = [FAKE] * 6 + [needd] + [FAKE] * 7 + [None]
assert len(args) == 15
assert lib.dma_attn_bwd(ctypes.byref(pd), *args) == UNSUPPORTED
args_bad = [FAKE] * 6 + [need] + [FAKE] * 6 + [None, None]
assert len(args_bad) == 15
assert lib.dma_attn_bwd(pp, *args_bad) == INVALID
# gate_bwd(p, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate, ws, ws_bytes, stream)
assert lib.dma_gate_bwd(pp, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == INVALID
# gate_bwd_noalloc(p, V, Delta, A, x_save, delta, d_delta, dDelta, dA, dV_gate, stream)
assert lib.dma_gate_bwd_noalloc(pp, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, None) == INVALID
pf = dma.make_params(1, 2, 1, 256, 64, 64, forward_only=True)   # forward-only: no backward
args = [FAKE] * 6 + [need_of(pf)] + [FAKE] * 7 + [None]
assert lib.dma_attn_bwd(ctypes.byref(pf), *args) == UNSUPPORTED
pc = dma.make_params(1, 2, 1, 256, 64, 64, Nq=100)   # chunked prefill: no backward
args = [FAKE] * 6 + [need_of(pc)] + [FAKE] * 7 + [None]
assert lib.dma_attn_bwd(ctypes.byref(pc), *args) == UNSUPPORTED
# topk_append(p, delta, ws, ws_bytes, stream): decode parameters only, a workspace of the plan's size
assert lib.dma_topk_append(pp, FAKE, FAKE, need, None) == INVALID
assert lib.dma_topk_append(ctypes.byref(pd), None, FAKE, needd, None) == INVALID
assert lib.dma_topk_append(ctypes.byref(pd), FAKE, FAKE, needd - 1, None) == WORKSPACE
# selftest_bounded_wait(p, ws, ws_bytes, limit_cycles, stream): the limit is checked first
assert lib.dma_selftest_bounded_wait(pp, FAKE, need, 0, None) == INVALID
assert lib.dma_selftest_bounded_wait(pp, FAKE, need, 1 << 40, None) == INVALID
assert lib.dma_selftest_bounded_wait(pp, FAKE, need - 1, 1000, None) == WORKSPACE
# gate_append(p, V, Delta, A, delta, x_save, stream)
assert lib.dma_gate_append(ctypes.byref(pd), FAKE, FAKE, FAKE, None, None, None) == INVALID
assert lib.dma_gate_append(ctypes.byref(pd), FAKE, FAKE, FAKE, FAKE, FAKE + 4, None) == INVALID
# context-parallel prefill: layout arguments, buffer sizes and workspace checked on the host
pc2 = dma.make_params(1, 4, 2, 500, 128, 64)
lay = dma._lib.DmaCpLayout()
assert lib.dma_cp_layout(ctypes.byref(pc2), 100, 0, ctypes.byref(lay)) == INVALID      # a prefix needs shards
assert lib.dma_cp_layout(ctypes.byref(pc2), 0, 1, ctypes.byref(lay)) == INVALID
assert lib.dma_cp_layout(ctypes.byref(pc2), 1000, 2, ctypes.byref(lay)) == OK and lay.prefix_rows == 128
assert lib.dma_cp_layout(ctypes.byref(pc2), 90, 1, ctypes.byref(lay)) == OK and lay.prefix_rows == 90
big = dma.make_params(1, 8, 1, 500, 128, 4096)                                      # G w = 32768 > 16384
assert lib.dma_cp_layout(ctypes.byref(big), 0, 0, ctypes.byref(lay)) == UNSUPPORTED
assert lib.dma_cp_layout(ctypes.byref(pc2), 0, 0, ctypes.byref(lay)) == OK
cb, wb = lay.cand_bytes, lay.ws_bytes
assert cb == 1024 + 1024 + 2 * (4 * 64 * 128 * 2)   # pos, delta, K rows, V rows of B H w = 4 x 64 entries
assert lib.dma_cp_candidates(ctypes.byref(pc2), 0, FAKE, FAKE, FAKE, FAKE, cb - 1, FAKE, wb, None) == INVALID
assert lib.dma_cp_candidates(ctypes.byref(pc2), 0, FAKE, FAKE, FAKE, FAKE, cb, FAKE, wb - 1, None) == WORKSPACE
assert lib.dma_cp_candidates(ctypes.byref(pc2), -1, FAKE, FAKE, FAKE, FAKE, cb, FAKE, wb, None) == INVALID
assert lib.dma_cp_compact(ctypes.byref(pc2), 1000, 2, FAKE, 2 * cb - 1, *([FAKE] * 7), FAKE, 1 << 30, None) == INVALID
assert lib.dma_cp_compact(ctypes.byref(pc2), 1000, 2, None, 2 * cb, *([FAKE] * 7), FAKE, 1 << 30, None) == INVALID
pdec = dma.make_params(8, 32, 8, 65536, 128, 2048, Nq=1)   # 64 MiB of gx alone: more than the fixed array
assert lib.dma_gate_bwd_noalloc(ctypes.byref(pdec), *([FAKE] * 9), None) == UNSUPPORTED
# the gate kernels hold at most 64 query heads; more is refused on the host, not at launch
ph = dma.make_params(1, 72, 8, 256, 128, 64)
needh = need_of(ph)
assert lib.dma_gate(ctypes.byref(ph), FAKE, FAKE, FAKE, FAKE, None, None, 0, None) == UNSUPPORTED
assert lib.dma_gate_bwd(ctypes.byref(ph), *([FAKE] * 9), FAKE, needh, None) == UNSUPPORTED
assert lib.dma_gate_bwd_noalloc(ctypes.byref(ph), *([FAKE] * 9), None) == UNSUPPORTED
# the scratch formula of dma_gate_bwd_noalloc, exact at the boundary of the fixed array: a problem that
# fits passes every host check and only fails for want of a device (DMA_ERR_CUDA), one more position
# does not fit (DMA_ERR_UNSUPPORTED)
CUDA_ERR = 4
a256 = lambda x: (x + 255) // 256 * 256
cdiv = lambda x, y: (x + y - 1) // y
def scratch(B, H, Hkv, N, d):
    return a256(4 * B * H * N) + a256(4 * B * H * cdiv(N, 1024)) + a256(4 * cdiv(N, 512) * B * Hkv * d * H)
LIMIT = 16 << 20
found = 0
for (B, H, Hkv, d) in ((1, 64, 8, 64), (3, 40, 8, 64), (2, 64, 4, 128)):
    lo, hi = 1, 1 << 24   # largest N whose scratch fits
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if scratch(B, H, Hkv, mid, d) <= LIMIT: lo = mid
        else: hi = mid - 1
    for N, want in ((lo, CUDA_ERR), (lo + 1, UNSUPPORTED)):
        q = dma.make_params(B, H, Hkv, N, d, 64, Nq=1)
        got = lib.dma_gate_bwd_noalloc(ctypes.byref(q), *([FAKE] * 9), None)
        assert got == want, (B, H, Hkv, d, N, got, want)
    found += 1
assert found == 3
print("ok")
"""


def test_null_and_misaligned_pointers_are_rejected_before_launch():
    import subprocess
    import sys
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", _FAKE_CHECKS % {"root": ROOT}], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr


def test_python_binding_raises_on_error_status():
    p = dma.make_params(1, 2, 1, 256, 64, 0)
    with pytest.raises(dma.DmaError, match="INVALID_ARG"):
        dma.workspace_size(p)
