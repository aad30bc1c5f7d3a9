"""Helpers for the GPU parity tests: device upload of the seeded inputs and the
comparison rules (attention tolerance, exact codes with counted rounding ties)."""
from __future__ import annotations

import numpy as np
import torch

import workloads as WL

ATOL_ABS = 1e-5
RTOL_MAX = 1e-3


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def q_tensor(q_bits: np.ndarray, q_dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).cuda()
    return t.view(torch.float16 if q_dtype == "fp16" else torch.bfloat16)


def decode_tensors(d: WL.DecodeInputs) -> dict:
    return dict(
        q=q_tensor(d.q_bits, d.w.q_dtype),
        lat_k=dev(d.lat_k), lat_v=dev(d.lat_v),
        scale_k=dev(d.scale_k), scale_v=dev(d.scale_v),
        B_k=dev(d.Bk), B_v=dev(d.Bv),
        seq_lens=dev(d.seq_lens),
    )


def assert_attention_close(gpu: np.ndarray, ref: np.ndarray, what: str = "", per_head: bool = True) -> float:
    """max|gpu - ref| <= 1e-3 * max|ref| + 1e-5, per (b, h) output vector.
    Returns the worst ratio error / allowance."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    if per_head:
        err = np.abs(gpu - ref).max(axis=-1)
        allow = RTOL_MAX * np.abs(ref).max(axis=-1) + ATOL_ABS
    else:
        err = np.abs(gpu - ref).max()
        allow = RTOL_MAX * np.abs(ref).max() + ATOL_ABS
    worst = float(np.max(err / allow))
    assert worst <= 1.0, f"{what}: error {worst:.3f}x the allowance (max err {np.max(err):.3e})"
    return worst


def _fp16_neighbours(x32: np.ndarray):
    """The two fp16 values bracketing each float32 value, and their midpoint."""
    h = x32.astype(np.float16)
    hf = h.astype(np.float32)
    up = np.nextafter(h, np.float16(np.inf)).astype(np.float32)
    dn = np.nextafter(h, np.float16(-np.inf)).astype(np.float32)
    lo = np.where(hf <= x32, hf, dn)
    hi = np.where(hf <= x32, up, hf)
    return lo, hi, (lo.astype(np.float64) + hi.astype(np.float64)) / 2


def compare_codes(g_codes, g_scale, o_codes, o_scale, o_c, bits: int, tie_tol: float = 1e-3,
                  scale_tol: float = 2.0 ** -20, stats: dict = None):
    """Codes must match the oracle exactly except +-1 at counted rounding ties.

    A code tie: the oracle's float32 ratio v = c / scale has |frac(|v|) - 0.5| <=
    tie_tol.  A scale tie: the oracle's float32 max|c| / Q lies within scale_tol
    (relative; 2^-20 for the fp32 paths) of an fp16 rounding midpoint; then the
    GPU scale may be the other neighbour and every code of that row may move by
    +-1.  `stats`, if given, collects the largest distance to the tie of every
    accepted mismatch ("scale_dist" relative, "code_dist" in code units): a
    measure of the kernel's error.
    Returns (n_code_ties, n_scale_ties)."""
    Q = 127 if bits == 8 else 7
    g_codes = np.asarray(g_codes, np.int64).reshape(-1, np.shape(g_codes)[-1])
    o_codes = np.asarray(o_codes, np.int64).reshape(g_codes.shape)
    g_scale = np.asarray(g_scale, np.float16).reshape(-1)
    o_scale = np.asarray(o_scale, np.float16).reshape(-1)
    c32 = np.asarray(o_c, np.float64).reshape(g_codes.shape).astype(np.float32)
    same_scale = g_scale.view(np.uint16) == o_scale.view(np.uint16)
    n_scale_ties = 0
    if not np.all(same_scale):
        amax = np.abs(c32).max(axis=1)
        ratio = (amax / np.float32(Q)).astype(np.float32)
        lo, hi, mid = _fp16_neighbours(ratio)
        bad = np.nonzero(~same_scale)[0]
        for i in bad:
            dist = abs(float(ratio[i]) - mid[i]) / max(abs(float(ratio[i])), 1e-30)
            if stats is not None:
                stats["scale_dist"] = max(stats.get("scale_dist", 0.0), dist)
            near = dist <= scale_tol
            other_ok = float(g_scale[i]) in (float(lo[i]), float(hi[i]))
            assert near and other_ok, f"row {i}: scale {g_scale[i]} vs oracle {o_scale[i]} is not a rounding tie"
            assert np.all(np.abs(g_codes[i] - o_codes[i]) <= 1), f"row {i}: codes off by more than 1"
        n_scale_ties = len(bad)
    rows = np.nonzero(same_scale)[0]
    d = g_codes[rows] - o_codes[rows]
    mism = np.nonzero(d)
    n_code_ties = 0
    if mism[0].size:
        s32 = o_scale[rows].astype(np.float32)[:, None]
        v = np.where(s32 > 0, c32[rows] / np.where(s32 > 0, s32, 1), 0).astype(np.float64)
        frac = np.abs(np.abs(v) - np.floor(np.abs(v)) - 0.5)
        if stats is not None:
            stats["code_dist"] = max(stats.get("code_dist", 0.0), float(frac[mism].max()))
        for i, j in zip(*mism):
            assert abs(d[i, j]) == 1 and frac[i, j] <= tie_tol, \
                f"row {rows[i]} col {j}: gpu {g_codes[rows[i], j]} oracle {o_codes[rows[i], j]} v={v[i, j]!r}"
        n_code_ties = int(mism[0].size)
    return n_code_ties, n_scale_ties


def unpack(lat: np.ndarray, r: int, bits: int) -> np.ndarray:
    """Cache bytes -> codes (test-side reader of the storage format)."""
    lat = np.asarray(lat, np.uint8)
    if bits == 8:
        return lat.view(np.int8).astype(np.int64)
    lo = (lat & 0xF).astype(np.int64)
    hi = (lat >> 4).astype(np.int64)
    out = np.empty(lat.shape[:-1] + (r,), np.int64)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out
