"""Seeded synthetic inputs for the WSVD low-rank decode path.

This module is shared by the tests, the float64 oracle's callers and the
benchmark.  It holds random draws, storage formats and workload shapes only:
no attention, projection or Hadamard arithmetic lives here.  Latent caches are
synthesised the way the workloads are stated ("latents ~N(0,1) stored as int8
/ packed int4 with a per-token-per-head fp16 scale max|x|/Q"); that storage step
is an input recipe and neither side of a parity test re-uses it.

Every block of random numbers is drawn from its own PCG64 stream keyed by
(seed, tensor id, b, h), so a test can regenerate one (b, h) slice of a
full-size workload without drawing the rest.

Layouts (all C-contiguous, the same ones the C-ABI takes):
  q            [B][H][Hd]            fp16 or bf16 (kept here as exact float32 + raw uint16 bits)
  lat_k, lat_v [B][H][L_cap][r*bits/8] uint8: int8 two's complement, or int4 with
                                     element 2j in bits 0-3 and 2j+1 in bits 4-7
  scale_k/v    [B][H][L_cap]         fp16
  Bk, Bv       [H][r][Hd]            fp16   (W_Kh ~= A_Kh . B_Kh)
  A_k, A_v     [H][E][r]             fp16
  x            [B][E]                bf16
  K, V (dense) [B][H][L_cap][Hd]     fp16
  shared lat   [B][L_cap][R]         fp16, shared B [H][R][Hd] fp16
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np

# Tensor ids for the per-block random streams.
_T_Q, _T_LK, _T_LV, _T_BK, _T_BV, _T_LEN, _T_OUTL = 1, 2, 3, 4, 5, 6, 7
_T_X, _T_AK, _T_AV, _T_XOUT = 10, 11, 12, 13
_T_DK, _T_DV, _T_SK, _T_SV, _T_SBK, _T_SBV = 20, 21, 22, 23, 24, 25
_T_S2K, _T_S2V = 30, 31
_T_QM = 40


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *key])))


# ----------------------------------------------------------------------------- formats
def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bf16 (ties to even), returned as float32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Raw bf16 bit patterns of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def to_dtype_exact(a: np.ndarray, dtype: str) -> Tuple[np.ndarray, np.ndarray]:
    """Round float data to fp16/bf16; return (exact float32 values, raw uint16 bits)."""
    if dtype == "fp16":
        h = np.asarray(a, dtype=np.float32).astype(np.float16)
        return h.astype(np.float32), h.view(np.uint16)
    if dtype == "bf16":
        v = round_to_bf16(np.asarray(a, dtype=np.float32))
        return v, bf16_bits(v)
    raise ValueError(dtype)


def qmax(bits: int) -> int:
    return 127 if bits == 8 else 7


def row_bytes(r: int, bits: int) -> int:
    return r * bits // 8


def store_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Integer codes [..., r] -> cache bytes [..., r*bits/8] (storage format only)."""
    c = np.asarray(codes, dtype=np.int16)
    if bits == 8:
        return c.astype(np.int8).view(np.uint8)
    nib = (c & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def synth_latent_storage(x: np.ndarray, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Input recipe from the workload statement: per row scale = fp16(max|x|/Q),
    integer code = nearest integer of x/scale, clipped to [-Q, Q].  Returns
    (cache bytes, fp16 scales)."""
    Q = qmax(bits)
    amax = np.abs(x).max(axis=-1)
    scale = (amax / Q).astype(np.float16)
    s = scale.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        codes = np.where(s > 0, np.rint(x / np.where(s > 0, s, 1.0)), 0.0)
    codes = np.clip(codes, -Q, Q).astype(np.int16)
    return store_codes(codes, bits), scale


# ----------------------------------------------------------------------------- shapes
@dataclass(frozen=True)
class Workload:
    """One synthetic workload.  `lens` is either a fixed length or an inclusive
    (lo, hi) range drawn uniformly per sequence."""
    name: str
    B: int
    H: int
    Hd: int
    r: int
    bits: int
    L_cap: int
    lens: object  # int or (lo, hi)
    q_dtype: str = "fp16"
    latent: str = "normal"  # "normal" | "student_t_outliers"
    E: int = 4096
    hadamard_block: int = 128
    append_steps: int = 0
    x_outlier_frac: float = 0.0
    x_outlier_gain: float = 1.0
    R: int = 0  # shared-latent rank for the comparison paths (0 = not used)
    prefill_tokens: int = 0  # prompt block written by one prefill call (0 = not measured)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


PR1 = Workload("pr1 b1 h4 hd64 r16 L256 int8", B=1, H=4, Hd=64, r=16, bits=8, L_cap=256, lens=256,
               q_dtype="fp16", E=256)
LLAVA7B = Workload("llava7b-layer b1 h32 hd128 r32 L1600(576 vision+1024 text) int8 + append E4096",
                   B=1, H=32, Hd=128, r=32, bits=8, L_cap=1600, lens=1600, q_dtype="bf16",
                   E=4096, append_steps=1, prefill_tokens=576)
RAGGED = Workload("ragged b16 h32 hd128 r32 L~U[1024,4096] int4 student-t+outliers",
                  B=16, H=32, Hd=128, r=32, bits=4, L_cap=4096, lens=(1024, 4096), q_dtype="fp16",
                  latent="student_t_outliers")
LONG = {r: Workload(f"long b4 h32 hd128 L32768 r{r} int8 + 64 appends E4096", B=4, H=32, Hd=128, r=r,
                    bits=8, L_cap=32768, lens=32768, q_dtype="bf16", E=4096, append_steps=64,
                    x_outlier_frac=0.001, x_outlier_gain=50.0)
        for r in (16, 32, 64)}
CMP = {L: Workload(f"cmp b8 h32 hd128 L{L} wsvd-r32-int8 / dense-fp16 / shared-R512", B=8, H=32,
                   Hd=128, r=32, bits=8, L_cap=L, lens=L, q_dtype="fp16", R=512)
       for L in (2048, 8192)}

PRESETS = {"pr1": PR1, "llava7b": LLAVA7B, "ragged": RAGGED,
           "long_r16": LONG[16], "long_r32": LONG[32], "long_r64": LONG[64],
           "cmp_l2048": CMP[2048], "cmp_l8192": CMP[8192]}


# ----------------------------------------------------------------------------- draws
def seq_lens(w: Workload, seed: int = 0) -> np.ndarray:
    if isinstance(w.lens, tuple):
        lo, hi = w.lens
        return _rng(seed, _T_LEN).integers(lo, hi + 1, size=w.B).astype(np.int32)
    return np.full(w.B, int(w.lens), dtype=np.int32)


def query(w: Workload, seed: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """q [B][H][Hd] ~ N(0,1) in the workload's dtype -> (float32 exact, uint16 bits)."""
    q = _rng(seed, _T_Q).standard_normal((w.B, w.H, w.Hd), dtype=np.float32)
    return to_dtype_exact(q, w.q_dtype)


def multi_query(w: Workload, seed: int, Tq: int, Hq: int) -> Tuple[np.ndarray, np.ndarray]:
    """Queries of a grouped / multi-token decode, q [B][Tq][Hq][Hd] ~ N(0,1) in
    the workload's dtype -> (float32 exact, uint16 bits).  The cache of such a
    workload has w.H = Hkv latent heads."""
    q = _rng(seed, _T_QM).standard_normal((w.B, Tq, Hq, w.Hd), dtype=np.float32)
    return to_dtype_exact(q, w.q_dtype)


def _outlier_channels(w: Workload, seed: int) -> np.ndarray:
    """Student-t workloads: 1% of (head, channel) pairs get a x20 gain."""
    g = _rng(seed, _T_OUTL)
    mask = g.random((w.H, w.r)) < 0.01
    return np.where(mask, 20.0, 1.0)


def latent_block(w: Workload, seed: int, b: int, h: int, which: str,
                 gains: Optional[np.ndarray] = None) -> np.ndarray:
    """Float latents [L_cap][r] of one (b, h) for K ('k') or V ('v')."""
    tid = _T_LK if which == "k" else _T_LV
    g = _rng(seed, tid, b, h)
    if w.latent == "normal":
        x = g.standard_normal((w.L_cap, w.r))
    else:
        x = g.standard_t(3.0, size=(w.L_cap, w.r))
        if gains is None:
            gains = _outlier_channels(w, seed)
        x = x * gains[h][None, :]
    return x


def up_proj(w: Workload, seed: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """B_K, B_V [H][r][Hd] fp16 ~ N(0, 1/r)."""
    sd = 1.0 / np.sqrt(w.r)
    bk = (_rng(seed, _T_BK).standard_normal((w.H, w.r, w.Hd)) * sd).astype(np.float16)
    bv = (_rng(seed, _T_BV).standard_normal((w.H, w.r, w.Hd)) * sd).astype(np.float16)
    return bk, bv


def latent_cache_block(w: Workload, seed: int, b: int, h: int, gains=None):
    """(lat_k bytes, scale_k, lat_v bytes, scale_v) for one (b, h), every row filled."""
    lk, sk = synth_latent_storage(latent_block(w, seed, b, h, "k", gains), w.bits)
    lv, sv = synth_latent_storage(latent_block(w, seed, b, h, "v", gains), w.bits)
    return lk, sk, lv, sv


def poison_rows(lat: np.ndarray, scale: np.ndarray, start: int, bits: int) -> None:
    """Fill rows >= start with extreme codes and non-finite scales (in place)."""
    if start >= lat.shape[0]:
        return
    lat[start:] = 0x7F if bits == 8 else 0x77
    s = scale[start:]
    s[0::3] = np.float16(np.nan)
    s[1::3] = np.float16(np.inf)
    s[2::3] = np.float16(65504.0)


@dataclass
class DecodeInputs:
    w: Workload
    seq_lens: np.ndarray
    q: np.ndarray       # float32 exact values
    q_bits: np.ndarray  # uint16
    lat_k: np.ndarray
    scale_k: np.ndarray
    lat_v: np.ndarray
    scale_v: np.ndarray
    Bk: np.ndarray
    Bv: np.ndarray
    extra: dict = field(default_factory=dict)


def decode_inputs(w: Workload, seed: int = 0, poison: bool = False, lens=None) -> DecodeInputs:
    """Full WSVD decode inputs.  Rows >= len_b are zero (or poisoned)."""
    L = seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    q, qb = query(w, seed)
    rb = row_bytes(w.r, w.bits)
    lat_k = np.zeros((w.B, w.H, w.L_cap, rb), np.uint8)
    lat_v = np.zeros_like(lat_k)
    sk = np.zeros((w.B, w.H, w.L_cap), np.float16)
    sv = np.zeros_like(sk)
    gains = _outlier_channels(w, seed) if w.latent != "normal" else None
    for b in range(w.B):
        n = int(L[b])
        for h in range(w.H):
            a, s1, c, s2 = latent_cache_block(w, seed, b, h, gains)
            lat_k[b, h, :n], sk[b, h, :n] = a[:n], s1[:n]
            lat_v[b, h, :n], sv[b, h, :n] = c[:n], s2[:n]
            if poison:
                poison_rows(lat_k[b, h], sk[b, h], n, w.bits)
                poison_rows(lat_v[b, h], sv[b, h], n, w.bits)
    bk, bv = up_proj(w, seed)
    return DecodeInputs(w, L, q, qb, lat_k, sk, lat_v, sv, bk, bv)


# ----------------------------------------------------------------------------- append
@dataclass
class AppendInputs:
    w: Workload
    x: np.ndarray       # [steps][B][E] float32 exact bf16 values
    x_bits: np.ndarray  # uint16
    A_k: np.ndarray     # [H][E][r] fp16
    A_v: np.ndarray


def append_inputs(w: Workload, seed: int = 0, steps: Optional[int] = None) -> AppendInputs:
    """x ~ N(0,1) bf16 (with a fixed set of outlier channels when the workload has
    them); A_K, A_V ~ N(0, 1/E) fp16."""
    steps = max(1, w.append_steps) if steps is None else steps
    x = _rng(seed, _T_X).standard_normal((steps, w.B, w.E), dtype=np.float32)
    if w.x_outlier_frac > 0:
        n_out = max(1, int(round(w.x_outlier_frac * w.E)))
        ch = _rng(seed, _T_XOUT).choice(w.E, size=n_out, replace=False)
        x[..., ch] *= np.float32(w.x_outlier_gain)
    xv, xb = to_dtype_exact(x, "bf16")
    sd = 1.0 / np.sqrt(w.E)
    ak = (_rng(seed, _T_AK).standard_normal((w.H, w.E, w.r)) * sd).astype(np.float16)
    av = (_rng(seed, _T_AV).standard_normal((w.H, w.E, w.r)) * sd).astype(np.float16)
    return AppendInputs(w, xv, xb, ak, av)


def prefill_inputs(w: Workload, seed: int = 0, T: int = 576) -> AppendInputs:
    """A block of T new tokens per sequence for the prefill latent write: the
    append recipe drawn for T steps and laid out [B][T][E], so that token t of
    the block is the activation step t of successive appends would take
    (x has shape [B][T][E] here, not [steps][B][E])."""
    ai = append_inputs(w, seed, steps=T)
    return AppendInputs(w, np.ascontiguousarray(ai.x.transpose(1, 0, 2)),
                        np.ascontiguousarray(ai.x_bits.transpose(1, 0, 2)), ai.A_k, ai.A_v)


def latent_rotation(w: Workload, seed: int = 0, which: str = "k") -> np.ndarray:
    """Synthetic orthogonal latent rotations S2 [H][r][r] (float32): the Q
    factor of a Gaussian matrix per head, sign-fixed so that diag(R) > 0."""
    g = _rng(seed, _T_S2K if which == "k" else _T_S2V).standard_normal((w.H, w.r, w.r))
    out = np.empty_like(g)
    for h in range(w.H):
        q, rr = np.linalg.qr(g[h])
        out[h] = q * np.sign(np.diag(rr))[None, :]
    return out.astype(np.float32)


def quantize_weights_w8(Wf: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Input recipe of the int8-weight (W8) workloads: each weight matrix
    [H][K][N] (fp16) is stored as symmetric int8 with one fp32 scale per output
    column, scale[h][n] = max_k |W[h][k][n]| / 127 (1 for an all-zero column),
    code = clamp(round_half_even(W / scale), -127, 127)."""
    w = np.asarray(Wf, np.float32)
    scale = (np.abs(w).max(axis=1) / np.float32(127.0)).astype(np.float32)
    scale[scale == 0] = 1.0
    q = np.clip(np.rint(w / scale[:, None, :]), -127, 127).astype(np.int8)
    return q, scale


# ----------------------------------------------------------------------------- comparisons
def dense_block(w: Workload, seed: int, b: int, h: int) -> Tuple[np.ndarray, np.ndarray]:
    """Dense K, V [L_cap][Hd] fp16 ~ N(0,1) for one (b, h)."""
    k = _rng(seed, _T_DK, b, h).standard_normal((w.L_cap, w.Hd), dtype=np.float32).astype(np.float16)
    v = _rng(seed, _T_DV, b, h).standard_normal((w.L_cap, w.Hd), dtype=np.float32).astype(np.float16)
    return k, v


def dense_inputs(w: Workload, seed: int = 0, lens=None) -> dict:
    L = seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    q, qb = query(w, seed)
    K = np.zeros((w.B, w.H, w.L_cap, w.Hd), np.float16)
    V = np.zeros_like(K)
    for b in range(w.B):
        n = int(L[b])
        for h in range(w.H):
            k, v = dense_block(w, seed, b, h)
            K[b, h, :n], V[b, h, :n] = k[:n], v[:n]
    return dict(seq_lens=L, q=q, q_bits=qb, K=K, V=V)


def shared_inputs(w: Workload, seed: int = 0, lens=None) -> dict:
    """Shared latent [B][L_cap][R] fp16 ~ N(0,1); per-head B [H][R][Hd] ~ N(0, 1/R)."""
    assert w.R > 0
    L = seq_lens(w, seed) if lens is None else np.asarray(lens, dtype=np.int32)
    q, qb = query(w, seed)
    lk = np.zeros((w.B, w.L_cap, w.R), np.float16)
    lv = np.zeros_like(lk)
    for b in range(w.B):
        n = int(L[b])
        lk[b, :n] = _rng(seed, _T_SK, b).standard_normal((n, w.R), dtype=np.float32).astype(np.float16)
        lv[b, :n] = _rng(seed, _T_SV, b).standard_normal((n, w.R), dtype=np.float32).astype(np.float16)
    sd = 1.0 / np.sqrt(w.R)
    bk = (_rng(seed, _T_SBK).standard_normal((w.H, w.R, w.Hd)) * sd).astype(np.float16)
    bv = (_rng(seed, _T_SBV).standard_normal((w.H, w.R, w.Hd)) * sd).astype(np.float16)
    return dict(seq_lens=L, q=q, q_bits=qb, lat_k=lk, lat_v=lv, Bk=bk, Bv=bv)
