"""The decode entry point that allocates nothing (wsvd_decode_attention_noalloc).

It serves callers that cannot call cudaMalloc (a runtime whose device memory is
one pre-sized pool owned by another allocator, code where an allocation would
synchronise or fail): its scratch is a static device array inside the library.
Checked here through the C ABI against the workspace-taking entry point on
the same inputs, twice in a row (the array keeps the previous call's
contents), and against the size limit.  This file is collected last on
purpose; it must pass on its own in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, decode_tensors

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 2 << 20  # WSVD_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def lib():
    from rank_kv_cache_wsvd_b200 import build
    build.build()
    return W.load()


def _noalloc(lib, d: WL.DecodeInputs, t: dict, out: torch.Tensor, err: torch.Tensor) -> int:
    w = d.w
    qdt = W._lib.WSVD_DTYPE_FP16 if w.q_dtype == "fp16" else W._lib.WSVD_DTYPE_BF16
    return lib.wsvd_decode_attention_noalloc(
        w.B, w.H, w.Hd, w.r, w.bits, w.L_cap, t["seq_lens"].data_ptr(), t["q"].data_ptr(), qdt,
        t["lat_k"].data_ptr(), t["lat_v"].data_ptr(), t["scale_k"].data_ptr(), t["scale_v"].data_ptr(),
        t["B_k"].data_ptr(), t["B_v"].data_ptr(), ctypes.c_float(0.0), out.data_ptr(), err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name,w,launches", [
    ("llava7b", WL.LLAVA7B, 1),                                 # cluster path, no scratch traffic
    ("ragged-int4", WL.RAGGED.with_(B=6), 2),                   # persistent path: partials + counters in the scratch
    ("long-r64", WL.LONG[64].with_(B=2, L_cap=8192, lens=8192), 2),
])
def test_noalloc_matches_workspace_entry_point_twice(lib, name, w, launches):
    """Bit for bit the output of wsvd_decode_attention, on two calls in a row.
    The launch count pins which decode path each case covers: the split-L
    grid (2 launches) is the one that keeps partials and counters in the
    static array."""
    assert W.wsvd_decode_launch_count(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap) == launches
    d = WL.decode_inputs(w, seed=11)
    t = decode_tensors(d)
    ref = W.wsvd_decode_attention(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                                  t["seq_lens"], bits=w.bits).cpu().numpy()
    for call in range(2):
        out = torch.full((w.B, w.H, w.Hd), float("nan"), dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _noalloc(lib, d, t, out, err) == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        got = out.cpu().numpy()
        assert_attention_close(got, ref, f"{name} call {call}")
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), f"{name} call {call}: not bitwise equal"


_FRESH = r"""
import ctypes, sys
import numpy as np, torch
sys.path[:0] = [{root!r}, {tests!r}]
import rank_kv_cache_wsvd_b200 as W, workloads as WL
from gpu_util import decode_tensors
lib = W.load()
torch.cuda.set_device(0)
w = WL.RAGGED.with_(B=3)
d = WL.decode_inputs(w, seed=5)
t = decode_tensors(d)
out = torch.full((w.B, w.H, w.Hd), float("nan"), dtype=torch.float32, device="cuda")
# the process's first library call is the no-allocation entry point
st = lib.wsvd_decode_attention_noalloc(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap, t["seq_lens"].data_ptr(),
    t["q"].data_ptr(), 0, t["lat_k"].data_ptr(), t["lat_v"].data_ptr(), t["scale_k"].data_ptr(),
    t["scale_v"].data_ptr(), t["B_k"].data_ptr(), t["B_v"].data_ptr(), ctypes.c_float(0.0), out.data_ptr(), None,
    torch.cuda.current_stream().cuda_stream)
assert st == 0, st
ref = W.wsvd_decode_attention(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                              t["seq_lens"], bits=w.bits)
torch.cuda.synchronize()
assert torch.equal(out, ref)
print("fresh-process noalloc ok")
"""


def test_noalloc_as_the_first_call_of_a_fresh_process(lib):
    """The per-device address lookup of the static array, made by the first
    call in a process that has not used the library before (one device)."""
    import os
    import subprocess
    import sys
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _FRESH.format(root=os.path.dirname(tests), tests=tests)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh-process noalloc ok" in r.stdout


def test_noalloc_rejects_problems_beyond_the_scratch_limit(lib):
    B, H, r = 64, 64, 128
    need = W.wsvd_decode_workspace_size(B, H, r)
    assert need > SCRATCH_LIMIT
    p = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = lib.wsvd_decode_attention_noalloc(B, H, 128, r, 8, 64, p, p, 0, p, p, p, p, p, p, ctypes.c_float(0.0), p,
                                           None, None)
    assert st == 4  # WSVD_ERR_WORKSPACE_TOO_SMALL
    assert lib.wsvd_status_string(st) == b"workspace too small"
