"""ctypes binding of libwsvd_b200.so: argument marshalling only.

Every operation runs in the library's CUDA kernels; PyTorch only provides
device memory and the current stream.  There is no CPU fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwsvd_b200.so")

WSVD_DTYPE_FP16 = 0
WSVD_DTYPE_BF16 = 1
DEVERR_LEN_RANGE = 1
DEVERR_CACHE_FULL = 2
DEVERR_PIPE_TIMEOUT = 4

_c_int, _c_size, _c_float, _p = ctypes.c_int, ctypes.c_size_t, ctypes.c_float, ctypes.c_void_p

# name -> (restype, argtypes); every symbol the public header declares.
SIGNATURES = {
    "wsvd_status_string": (ctypes.c_char_p, [_c_int]),
    "wsvd_abi_version": (_c_int, []),
    "wsvd_cache_bytes": (_c_size, [_c_int] * 5),
    "shared_cache_bytes": (_c_size, [_c_int] * 3),
    "dense_cache_bytes": (_c_size, [_c_int] * 4),
    "wsvd_decode_workspace_size": (_c_size, [_c_int] * 3),
    "dense_decode_workspace_size": (_c_size, [_c_int] * 3),
    "shared_decode_workspace_size": (_c_size, [_c_int] * 3),
    "wsvd_append_workspace_size": (_c_size, []),
    "wsvd_decode_launch_count": (_c_int, [_c_int] * 6),
    "wsvd_step_launch_count": (_c_int, [_c_int] * 9),
    "wsvd_decode_attention": (_c_int, [_c_int] * 6 + [_p, _p, _c_int] + [_p] * 6 + [_c_float, _p, _p, _c_size,
                                                                                        _p, _p]),
    "wsvd_decode_attention_noalloc": (_c_int, [_c_int] * 6 + [_p, _p, _c_int] + [_p] * 6 + [_c_float, _p, _p, _p]),
    "wsvd_latent_append": (_c_int, [_c_int] * 7 + [_p, _c_int] + [_p] * 7 + [_p, _c_size, _p, _p]),
    "wsvd_prefill_workspace_size": (_c_size, [_c_int] * 3),
    "wsvd_latent_prefill": (_c_int, [_c_int] * 8 + [_p, _c_int, _p, _p] + [_p] * 5 + [_p, _c_size, _p, _p]),
    "wsvd_append_and_decode": (_c_int, [_c_int] * 8 + [_p, _c_int, _p, _p] + [_p] * 5 + [_p, _c_int, _p, _p]
                               + [_c_float, _p, _p, _c_size, _p, _c_size, _p, _p]),
    "wsvd_decode_multi_workspace_size": (_c_size, [_c_int] * 6),
    "wsvd_decode_multi": (_c_int, [_c_int] * 8 + [_p, _p, _c_int] + [_p] * 6 + [_c_float, _p, _p, _c_size, _p, _p]),
    "wsvd_decode_gqa_workspace_size": (_c_size, [_c_int] * 5),
    "wsvd_decode_gqa": (_c_int, [_c_int] * 7 + [_p, _p, _c_int] + [_p] * 6 + [_c_float, _p, _p, _c_size, _p, _p]),
    "wsvd_step_host_workspace_size": (_c_size, [_c_int] * 5),
    "wsvd_append_and_decode_host": (_c_int, [_c_int] * 8 + [_p, _c_int, _p, _p] + [_p] * 5 + [_p, _c_int, _p, _p]
                                    + [_c_float, _p, _p, _c_size, _p, _p]),
    "wsvd_step_host_graph_create": (_c_int, [_c_int] * 8 + [_p, _c_int, _p, _p] + [_p] * 5 + [_p, _c_int, _p, _p]
                                    + [_c_float, _p, _p, _c_size, _p, _p]),
    "wsvd_step_host_graph_launch": (_c_int, [_p, _p]),
    "wsvd_step_host_graph_destroy": (None, [_p]),
    "wsvd_decode_attention_w8": (_c_int, [_c_int] * 6 + [_p, _p, _c_int] + [_p] * 8 + [_c_float, _p, _p, _c_size,
                                                                                           _p, _p]),
    "wsvd_latent_append_w8": (_c_int, [_c_int] * 7 + [_p, _c_int] + [_p] * 9 + [_p, _c_size, _p, _p]),
    "wsvd_append_and_decode_w8": (_c_int, [_c_int] * 8 + [_p, _c_int] + [_p] * 9 + [_p, _c_int] + [_p] * 4
                                  + [_c_float, _p, _p, _c_size, _p, _c_size, _p, _p]),
    "wsvd_fold_latent_rotation": (_c_int, [_c_int] * 4 + [_p] * 11),
    "dense_decode_attention": (_c_int, [_c_int] * 4 + [_p, _p, _c_int, _p, _p, _c_float, _p, _p, _c_size, _p, _p]),
    "shared_latent_svd_decode": (_c_int, [_c_int] * 5 + [_p, _p, _c_int] + [_p] * 4 + [_c_float, _p, _p, _c_size,
                                                                                         _p, _p]),
}

_lib = None


class WsvdError(RuntimeError):
    pass


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise WsvdError(f"{path} is missing: build it with `python -m rank_kv_cache_wsvd_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != 0:
        msg = load().wsvd_status_string(status).decode()
        raise WsvdError(f"{what}: {msg} (status {status})")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise WsvdError("all tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise WsvdError("all tensors must be contiguous")
    return t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return WSVD_DTYPE_FP16
    if t.dtype == torch.bfloat16:
        return WSVD_DTYPE_BF16
    raise WsvdError(f"expected fp16 or bf16, got {t.dtype}")


def _expect(t: torch.Tensor, dtype, shape, name: str) -> None:
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise WsvdError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


# ----------------------------------------------------------------------------- sizes
def wsvd_cache_bytes(B, H, L_cap, r, bits) -> int:
    return load().wsvd_cache_bytes(B, H, L_cap, r, bits)


def shared_cache_bytes(B, L_cap, R) -> int:
    return load().shared_cache_bytes(B, L_cap, R)


def dense_cache_bytes(B, H, L_cap, Hd) -> int:
    return load().dense_cache_bytes(B, H, L_cap, Hd)


def wsvd_decode_workspace_size(B, H, r) -> int:
    return load().wsvd_decode_workspace_size(B, H, r)


def wsvd_decode_launch_count(B, H, Hd, r, bits, L_cap) -> int:
    """Kernels one wsvd_decode_attention call with these sizes launches on the current device."""
    return load().wsvd_decode_launch_count(B, H, Hd, r, bits, L_cap)


def wsvd_step_launch_count(B, H, Hd, E, r, bits, L_cap, hadamard_block=128, w8=False) -> int:
    """Kernels one wsvd_append_and_decode(_w8) call with these sizes launches on
    the current device: 1 when the append and the decode run as one kernel."""
    return load().wsvd_step_launch_count(B, H, Hd, E, r, bits, L_cap, hadamard_block, int(bool(w8)))


def dense_decode_workspace_size(B, H, Hd) -> int:
    return load().dense_decode_workspace_size(B, H, Hd)


def shared_decode_workspace_size(B, H, R) -> int:
    return load().shared_decode_workspace_size(B, H, R)


def wsvd_append_workspace_size() -> int:
    return load().wsvd_append_workspace_size()


def wsvd_prefill_workspace_size(B, T, E) -> int:
    return load().wsvd_prefill_workspace_size(B, T, E)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Caller-owned scratch buffer (uint8), zero-filled."""
    return torch.zeros(max(16, nbytes), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------------------- decode
def wsvd_decode_attention(q, lat_k, lat_v, scale_k, scale_v, B_k, B_v, seq_lens, bits: int,
                          softmax_scale: float = 0.0, out=None, workspace_buf=None, err=None, stream=None):
    """Decode step over a per-head low-rank cache; returns out [B][H][Hd] fp32."""
    lib = load()
    B, H, Hd = q.shape
    L_cap, rb = lat_k.shape[2], lat_k.shape[3]
    r = rb * 8 // bits
    _expect(lat_k, torch.uint8, (B, H, L_cap, rb), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, rb), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(B_k, torch.float16, (H, r, Hd), "B_k")
    _expect(B_v, torch.float16, (H, r, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, H, Hd), "out")
    need = lib.wsvd_decode_workspace_size(B, H, r)
    if workspace_buf is None:
        workspace_buf = workspace(need, q.device)
    st = lib.wsvd_decode_attention(B, H, Hd, r, bits, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q),
                                   _ptr(lat_k), _ptr(lat_v), _ptr(scale_k), _ptr(scale_v), _ptr(B_k), _ptr(B_v),
                                   float(softmax_scale), _ptr(out), _ptr(workspace_buf), workspace_buf.numel(),
                                   _ptr(err), _stream(stream))
    _check(st, "wsvd_decode_attention")
    return out


def wsvd_decode_multi_workspace_size(B, Tq, Hq, Hkv, r, L_cap) -> int:
    return load().wsvd_decode_multi_workspace_size(B, Tq, Hq, Hkv, r, L_cap)


def wsvd_decode_multi(q, lat_k, lat_v, scale_k, scale_v, B_k, B_v, seq_lens, bits: int,
                      softmax_scale: float = 0.0, out=None, workspace_buf=None, err=None, stream=None):
    """Grouped / multi-token decode: q [B][Tq][Hq][Hd] over a cache of Hkv latent
    heads (query head g reads latent head g // (Hq // Hkv)); query token t
    sees rows [0, seq_lens[b] - Tq + 1 + t).  Returns out [B][Tq][Hq][Hd] fp32."""
    lib = load()
    B, Tq, Hq, Hd = q.shape
    Hkv, L_cap, rb = lat_k.shape[1], lat_k.shape[2], lat_k.shape[3]
    r = rb * 8 // bits
    _expect(lat_k, torch.uint8, (B, Hkv, L_cap, rb), "lat_k")
    _expect(lat_v, torch.uint8, (B, Hkv, L_cap, rb), "lat_v")
    _expect(scale_k, torch.float16, (B, Hkv, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, Hkv, L_cap), "scale_v")
    _expect(B_k, torch.float16, (Hkv, r, Hd), "B_k")
    _expect(B_v, torch.float16, (Hkv, r, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, Tq, Hq, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, Tq, Hq, Hd), "out")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_decode_multi_workspace_size(B, Tq, Hq, Hkv, r, L_cap), q.device)
    st = lib.wsvd_decode_multi(B, Tq, Hq, Hkv, Hd, r, bits, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q),
                               _ptr(lat_k), _ptr(lat_v), _ptr(scale_k), _ptr(scale_v), _ptr(B_k), _ptr(B_v),
                               float(softmax_scale), _ptr(out), _ptr(workspace_buf), workspace_buf.numel(), _ptr(err),
                               _stream(stream))
    _check(st, "wsvd_decode_multi")
    return out


def wsvd_decode_gqa(q, lat_k, lat_v, scale_k, scale_v, B_k, B_v, seq_lens, bits: int, softmax_scale: float = 0.0,
                    out=None, workspace_buf=None, err=None, stream=None):
    """Grouped-query decode: q [B][Hq][Hd] over Hkv latent heads; out [B][Hq][Hd] fp32."""
    lib = load()
    B, Hq, Hd = q.shape
    Hkv, L_cap, rb = lat_k.shape[1], lat_k.shape[2], lat_k.shape[3]
    r = rb * 8 // bits
    _expect(lat_k, torch.uint8, (B, Hkv, L_cap, rb), "lat_k")
    _expect(lat_v, torch.uint8, (B, Hkv, L_cap, rb), "lat_v")
    _expect(scale_k, torch.float16, (B, Hkv, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, Hkv, L_cap), "scale_v")
    _expect(B_k, torch.float16, (Hkv, r, Hd), "B_k")
    _expect(B_v, torch.float16, (Hkv, r, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, Hq, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, Hq, Hd), "out")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_decode_gqa_workspace_size(B, Hq, Hkv, r, L_cap), q.device)
    st = lib.wsvd_decode_gqa(B, Hq, Hkv, Hd, r, bits, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q), _ptr(lat_k),
                             _ptr(lat_v), _ptr(scale_k), _ptr(scale_v), _ptr(B_k), _ptr(B_v), float(softmax_scale),
                             _ptr(out), _ptr(workspace_buf), workspace_buf.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_decode_gqa")
    return out


def dense_decode_attention(q, K, V, seq_lens, softmax_scale: float = 0.0, out=None, workspace_buf=None,
                           err=None, stream=None):
    lib = load()
    B, H, Hd = q.shape
    L_cap = K.shape[2]
    _expect(K, torch.float16, (B, H, L_cap, Hd), "K")
    _expect(V, torch.float16, (B, H, L_cap, Hd), "V")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    need = lib.dense_decode_workspace_size(B, H, Hd)
    if workspace_buf is None:
        workspace_buf = workspace(need, q.device)
    st = lib.dense_decode_attention(B, H, Hd, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q), _ptr(K), _ptr(V),
                                    float(softmax_scale), _ptr(out), _ptr(workspace_buf), workspace_buf.numel(),
                                    _ptr(err), _stream(stream))
    _check(st, "dense_decode_attention")
    return out


def shared_latent_svd_decode(q, lat_k, lat_v, B_k, B_v, seq_lens, softmax_scale: float = 0.0, out=None,
                             workspace_buf=None, err=None, stream=None):
    lib = load()
    B, H, Hd = q.shape
    L_cap, R = lat_k.shape[1], lat_k.shape[2]
    _expect(lat_k, torch.float16, (B, L_cap, R), "lat_k")
    _expect(lat_v, torch.float16, (B, L_cap, R), "lat_v")
    _expect(B_k, torch.float16, (H, R, Hd), "B_k")
    _expect(B_v, torch.float16, (H, R, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    need = lib.shared_decode_workspace_size(B, H, R)
    if workspace_buf is None:
        workspace_buf = workspace(need, q.device)
    st = lib.shared_latent_svd_decode(B, H, Hd, R, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q), _ptr(lat_k),
                                      _ptr(lat_v), _ptr(B_k), _ptr(B_v), float(softmax_scale), _ptr(out),
                                      _ptr(workspace_buf), workspace_buf.numel(), _ptr(err), _stream(stream))
    _check(st, "shared_latent_svd_decode")
    return out


# ----------------------------------------------------------------------------- one step
def wsvd_append_and_decode(x, A_k, A_v, seq_lens, lat_k, lat_v, scale_k, scale_v, q, B_k, B_v, bits: int,
                           hadamard_block: int = 128, softmax_scale: float = 0.0, out=None, append_ws=None,
                           decode_ws=None, err=None, stream=None):
    """Append the new token's latents, then decode over the cache including it
    (one library call; the decode overlaps the append's tail).  Returns out
    [B][H][Hd] fp32; seq_lens and the cache are updated in place."""
    lib = load()
    B, E = x.shape
    H, _, r = A_k.shape
    Hd = q.shape[2]
    L_cap = lat_k.shape[2]
    _expect(A_k, torch.float16, (H, E, r), "A_k")
    _expect(A_v, torch.float16, (H, E, r), "A_v")
    _expect(q, q.dtype, (B, H, Hd), "q")
    _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(B_k, torch.float16, (H, r, Hd), "B_k")
    _expect(B_v, torch.float16, (H, r, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, H, Hd), "out")
    if append_ws is None:
        append_ws = workspace(lib.wsvd_append_workspace_size(), x.device)
    if decode_ws is None:
        decode_ws = workspace(lib.wsvd_decode_workspace_size(B, H, r), q.device)
    st = lib.wsvd_append_and_decode(B, H, Hd, E, r, bits, L_cap, hadamard_block, _ptr(x), _dtype_code(x),
                                    _ptr(A_k), _ptr(A_v), _ptr(seq_lens), _ptr(lat_k), _ptr(lat_v), _ptr(scale_k),
                                    _ptr(scale_v), _ptr(q), _dtype_code(q), _ptr(B_k), _ptr(B_v),
                                    float(softmax_scale), _ptr(out), _ptr(append_ws), append_ws.numel(),
                                    _ptr(decode_ws), decode_ws.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_append_and_decode")
    return out


def wsvd_step_host_workspace_size(B, H, Hd, E, r) -> int:
    return load().wsvd_step_host_workspace_size(B, H, Hd, E, r)


class StepFromHost:
    """One decode step whose per-step inputs and output are host buffers:
    wsvd_append_and_decode_host with every argument checked and converted
    once, here, so that a call is one C call with no Python-side checks.

    x_host [B][E] and q_host [B][H][Hd] (16-bit) and out_host [B][H][Hd]
    fp32 are CPU tensors, ideally pinned; the device tensors (weights, cache,
    seq_lens) are bound as given.  After `__call__` the step is queued on the
    stream given here; out_host is valid once that stream is synchronised,
    and x_host, q_host may be rewritten for the next step only after that.
    With `graph` (the default when all three host buffers are pinned) the
    step's launches are captured once into a CUDA graph
    (wsvd_step_host_graph_create) and a call is one graph launch.  The caller
    keeps every bound tensor alive and unchanged in shape."""

    def __init__(self, x_host, A_k, A_v, seq_lens, lat_k, lat_v, scale_k, scale_v, q_host, B_k, B_v, out_host,
                 bits: int, hadamard_block: int = 128, softmax_scale: float = 0.0, err=None, stream=None,
                 graph=None):
        lib = load()
        B, E = x_host.shape
        H, _, r = A_k.shape
        Hd = q_host.shape[2]
        L_cap = lat_k.shape[2]
        for t, name in ((x_host, "x_host"), (q_host, "q_host"), (out_host, "out_host")):
            if t.is_cuda or not t.is_contiguous():
                raise WsvdError(f"{name} must be a contiguous host tensor")
        _expect(out_host, torch.float32, (B, H, Hd), "out_host")
        _expect(q_host, q_host.dtype, (B, H, Hd), "q_host")
        _expect(A_k, torch.float16, (H, E, r), "A_k")
        _expect(A_v, torch.float16, (H, E, r), "A_v")
        _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
        _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
        _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
        _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
        _expect(B_k, torch.float16, (H, r, Hd), "B_k")
        _expect(B_v, torch.float16, (H, r, Hd), "B_v")
        _expect(seq_lens, torch.int32, (B,), "seq_lens")
        self.workspace = workspace(lib.wsvd_step_host_workspace_size(B, H, Hd, E, r), A_k.device)
        self._keep = (x_host, A_k, A_v, seq_lens, lat_k, lat_v, scale_k, scale_v, q_host, B_k, B_v, out_host, err)
        self.h2d_bytes = x_host.numel() * 2 + q_host.numel() * 2
        self.d2h_bytes = out_host.numel() * 4
        self._lib = lib
        self._fn = lib.wsvd_append_and_decode_host
        args = (B, H, Hd, E, r, bits, L_cap, hadamard_block, x_host.data_ptr(), _dtype_code(x_host),
                _ptr(A_k), _ptr(A_v), _ptr(seq_lens), _ptr(lat_k), _ptr(lat_v), _ptr(scale_k),
                _ptr(scale_v), q_host.data_ptr(), _dtype_code(q_host), _ptr(B_k), _ptr(B_v),
                float(softmax_scale), out_host.data_ptr(), _ptr(self.workspace), self.workspace.numel(),
                _ptr(err))
        self._args = args + (_stream(stream),)
        self._graph = None
        if graph is None:
            graph = x_host.is_pinned() and q_host.is_pinned() and out_host.is_pinned()
        if graph:
            handle = ctypes.c_void_p()
            st = lib.wsvd_step_host_graph_create(*args, ctypes.byref(handle))
            _check(st, "wsvd_step_host_graph_create")
            self._graph = handle
            self._launch = lib.wsvd_step_host_graph_launch
            self._gargs = (handle, _stream(stream))

    @property
    def uses_graph(self) -> bool:
        return self._graph is not None

    def __call__(self) -> None:
        if self._graph is not None:
            st = self._launch(*self._gargs)
            if st:
                _check(st, "wsvd_step_host_graph_launch")
            return
        st = self._fn(*self._args)
        if st:
            _check(st, "wsvd_append_and_decode_host")

    def close(self) -> None:
        """Releases the captured graph (no step of it may still be pending)."""
        if self._graph is not None:
            self._lib.wsvd_step_host_graph_destroy(self._graph)
            self._graph = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------------------- int8 weights
def _w8(t, s, shape_t, shape_s, name):
    _expect(t, torch.int8, shape_t, name)
    _expect(s, torch.float32, shape_s, "scales of " + name)


def wsvd_decode_attention_w8(q, lat_k, lat_v, scale_k, scale_v, B_k, B_v, sB_k, sB_v, seq_lens, bits: int,
                             softmax_scale: float = 0.0, out=None, workspace_buf=None, err=None, stream=None):
    """Decode with int8 B_k, B_v [H][r][Hd] and per-column fp32 scales [H][Hd]."""
    lib = load()
    B, H, Hd = q.shape
    L_cap, rb = lat_k.shape[2], lat_k.shape[3]
    r = rb * 8 // bits
    _expect(lat_k, torch.uint8, (B, H, L_cap, rb), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, rb), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _w8(B_k, sB_k, (H, r, Hd), (H, Hd), "B_k")
    _w8(B_v, sB_v, (H, r, Hd), (H, Hd), "B_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, H, Hd), "out")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_decode_workspace_size(B, H, r), q.device)
    st = lib.wsvd_decode_attention_w8(B, H, Hd, r, bits, L_cap, _ptr(seq_lens), _ptr(q), _dtype_code(q),
                                      _ptr(lat_k), _ptr(lat_v), _ptr(scale_k), _ptr(scale_v), _ptr(B_k), _ptr(B_v),
                                      _ptr(sB_k), _ptr(sB_v), float(softmax_scale), _ptr(out), _ptr(workspace_buf),
                                      workspace_buf.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_decode_attention_w8")
    return out


def wsvd_latent_append_w8(x, A_k, A_v, sA_k, sA_v, seq_lens, lat_k, lat_v, scale_k, scale_v, bits: int,
                          hadamard_block: int = 128, workspace_buf=None, err=None, stream=None) -> None:
    """Append with int8 A_k, A_v [H][E][r] and per-column fp32 scales [H][r]."""
    lib = load()
    B, E = x.shape
    H, _, r = A_k.shape
    L_cap = lat_k.shape[2]
    _w8(A_k, sA_k, (H, E, r), (H, r), "A_k")
    _w8(A_v, sA_v, (H, E, r), (H, r), "A_v")
    _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_append_workspace_size(), x.device)
    st = lib.wsvd_latent_append_w8(B, H, E, r, bits, L_cap, hadamard_block, _ptr(x), _dtype_code(x), _ptr(A_k),
                                   _ptr(A_v), _ptr(sA_k), _ptr(sA_v), _ptr(seq_lens), _ptr(lat_k), _ptr(lat_v),
                                   _ptr(scale_k), _ptr(scale_v), _ptr(workspace_buf), workspace_buf.numel(),
                                   _ptr(err), _stream(stream))
    _check(st, "wsvd_latent_append_w8")


def wsvd_append_and_decode_w8(x, A_k, A_v, sA_k, sA_v, seq_lens, lat_k, lat_v, scale_k, scale_v, q, B_k, B_v,
                              sB_k, sB_v, bits: int, hadamard_block: int = 128, softmax_scale: float = 0.0,
                              out=None, append_ws=None, decode_ws=None, err=None, stream=None):
    """wsvd_append_and_decode with int8 weights (A: [H][E][r] + [H][r] scales;
    B: [H][r][Hd] + [H][Hd] scales)."""
    lib = load()
    B, E = x.shape
    H, _, r = A_k.shape
    Hd = q.shape[2]
    L_cap = lat_k.shape[2]
    _w8(A_k, sA_k, (H, E, r), (H, r), "A_k")
    _w8(A_v, sA_v, (H, E, r), (H, r), "A_v")
    _w8(B_k, sB_k, (H, r, Hd), (H, Hd), "B_k")
    _w8(B_v, sB_v, (H, r, Hd), (H, Hd), "B_v")
    _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if out is None:
        out = torch.empty((B, H, Hd), dtype=torch.float32, device=q.device)
    _expect(out, torch.float32, (B, H, Hd), "out")
    if append_ws is None:
        append_ws = workspace(lib.wsvd_append_workspace_size(), x.device)
    if decode_ws is None:
        decode_ws = workspace(lib.wsvd_decode_workspace_size(B, H, r), q.device)
    st = lib.wsvd_append_and_decode_w8(B, H, Hd, E, r, bits, L_cap, hadamard_block, _ptr(x), _dtype_code(x),
                                       _ptr(A_k), _ptr(A_v), _ptr(sA_k), _ptr(sA_v), _ptr(seq_lens), _ptr(lat_k),
                                       _ptr(lat_v), _ptr(scale_k), _ptr(scale_v), _ptr(q), _dtype_code(q),
                                       _ptr(B_k), _ptr(B_v), _ptr(sB_k), _ptr(sB_v), float(softmax_scale),
                                       _ptr(out), _ptr(append_ws), append_ws.numel(), _ptr(decode_ws),
                                       decode_ws.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_append_and_decode_w8")
    return out


# ----------------------------------------------------------------------------- latent rotation
def wsvd_fold_latent_rotation(S2_k, S2_v, A_k, A_v, B_k, B_v, stream=None):
    """A' = A . S2 and B' = S2^T . B per head (weight preparation).  Returns
    (A_k', A_v', B_k', B_v') as new fp16 tensors."""
    lib = load()
    H, E, r = A_k.shape
    Hd = B_k.shape[2]
    for t, shape, name in ((S2_k, (H, r, r), "S2_k"), (S2_v, (H, r, r), "S2_v")):
        _expect(t, torch.float32, shape, name)
    for t, shape, name in ((A_k, (H, E, r), "A_k"), (A_v, (H, E, r), "A_v"), (B_k, (H, r, Hd), "B_k"),
                           (B_v, (H, r, Hd), "B_v")):
        _expect(t, torch.float16, shape, name)
    outs = [torch.empty_like(t) for t in (A_k, A_v, B_k, B_v)]
    st = lib.wsvd_fold_latent_rotation(H, E, r, Hd, _ptr(S2_k), _ptr(S2_v), _ptr(A_k), _ptr(A_v), _ptr(B_k),
                                       _ptr(B_v), *[_ptr(o) for o in outs], _stream(stream))
    _check(st, "wsvd_fold_latent_rotation")
    return tuple(outs)


# ----------------------------------------------------------------------------- append
def wsvd_latent_append(x, A_k, A_v, seq_lens, lat_k, lat_v, scale_k, scale_v, bits: int,
                       hadamard_block: int = 128, workspace_buf=None, err=None, stream=None) -> None:
    """Quantise one new token per sequence into the cache and advance seq_lens (in place).

    `workspace_buf` must be zero before its first use (the default allocation is);
    every call leaves it zero."""
    lib = load()
    B, E = x.shape
    H, _, r = A_k.shape
    L_cap, rb = lat_k.shape[2], lat_k.shape[3]
    _expect(A_k, torch.float16, (H, E, r), "A_k")
    _expect(A_v, torch.float16, (H, E, r), "A_v")
    _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_append_workspace_size(), x.device)
    st = lib.wsvd_latent_append(B, H, E, r, bits, L_cap, hadamard_block, _ptr(x), _dtype_code(x), _ptr(A_k),
                                _ptr(A_v), _ptr(seq_lens), _ptr(lat_k), _ptr(lat_v), _ptr(scale_k), _ptr(scale_v),
                                _ptr(workspace_buf), workspace_buf.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_latent_append")


def wsvd_latent_prefill(x, A_k, A_v, seq_lens, lat_k, lat_v, scale_k, scale_v, bits: int,
                        hadamard_block: int = 128, workspace_buf=None, err=None, stream=None) -> None:
    """Quantise a block of T new tokens per sequence (x [B][T][E]) into cache rows
    seq_lens[b] .. seq_lens[b] + T - 1 and advance seq_lens by T (in place)."""
    lib = load()
    B, T, E = x.shape
    H, _, r = A_k.shape
    L_cap = lat_k.shape[2]
    _expect(A_k, torch.float16, (H, E, r), "A_k")
    _expect(A_v, torch.float16, (H, E, r), "A_v")
    _expect(lat_k, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_k")
    _expect(lat_v, torch.uint8, (B, H, L_cap, r * bits // 8), "lat_v")
    _expect(scale_k, torch.float16, (B, H, L_cap), "scale_k")
    _expect(scale_v, torch.float16, (B, H, L_cap), "scale_v")
    _expect(seq_lens, torch.int32, (B,), "seq_lens")
    if workspace_buf is None:
        workspace_buf = workspace(lib.wsvd_prefill_workspace_size(B, T, E), x.device)
    st = lib.wsvd_latent_prefill(B, T, H, E, r, bits, L_cap, hadamard_block, _ptr(x), _dtype_code(x), _ptr(A_k),
                                 _ptr(A_v), _ptr(seq_lens), _ptr(lat_k), _ptr(lat_v), _ptr(scale_k), _ptr(scale_v),
                                 _ptr(workspace_buf), workspace_buf.numel(), _ptr(err), _stream(stream))
    _check(st, "wsvd_latent_prefill")
