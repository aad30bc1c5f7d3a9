"""Float64 CPU oracle for WSVD's low-rank, low-precision KV-cache decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this module
and the two share no code.  Only the tests, `__graft_entry__.smoke()` and the
CPU-baseline / reference leg of `bench.py` may import or run it.

Everything here is the plain definition, written for a reader to check by eye
against the WSVD summary pages ("WSVD: Weighted Low-Rank Approximation for Fast
and Efficient Execution of Low-Precision Vision-Language Models", gist.science
paper 2604.02570, summaries in ja / de / it / ar):

* per-head factorisation W_Kh ~= A_Kh . B_Kh with A_Kh in R^{E x r} and
  B_Kh in R^{r x Hd}; each head keeps its own L x r latent cache C_Kh
  (de §2.A "Fein granulare SVD pro Attention-Head"; ar §2.a);
* low-precision latents (W8A8 / W8A4) and the Hadamard rotation S1 applied to
  activations before quantisation (de §2.C "Quantisierungsbewusstes Training");
* the decode step rebuilds K and V from the latents and runs q.K^T, softmax and
  the V product (ja §2.4 "システム実装：融合カーネル"; de §2.D).  The oracle
  materialises K = lat_K . B_K and V = lat_V . B_V explicitly, which is exactly
  the reconstruction the fused GPU kernel avoids writing out.

All arithmetic is float64 except where a floating-point value decides an
integer (a quantised code, an fp16 scale): the pages fix no precision for that
decision, so it is taken in the kernel's float32, as the GPU does.

Pins: every function here is checked in tests/test_oracle_pins.py against brute
force on tiny inputs, closed forms, invariants and library routines.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np


# ----------------------------------------------------------------------------- codes
def qmax(bits: int) -> int:
    """Largest code magnitude of the symmetric quantiser: 127 for int8, 7 for int4
    (the int4 code -8 is never produced)."""
    if bits == 8:
        return 127
    if bits == 4:
        return 7
    raise ValueError(f"bits must be 8 or 4, got {bits}")


def unpack_codes(lat: np.ndarray, r: int, bits: int) -> np.ndarray:
    """Cache bytes [..., r*bits/8] -> integer codes [..., r].

    int8: two's complement bytes.  int4: element 2j in the low nibble and 2j+1
    in the high nibble of byte j, each a two's complement nibble."""
    lat = np.asarray(lat, dtype=np.uint8)
    if bits == 8:
        assert lat.shape[-1] == r
        return lat.view(np.int8).astype(np.int64)
    assert lat.shape[-1] * 2 == r
    out = np.empty(lat.shape[:-1] + (r,), dtype=np.int64)
    for j in range(r // 2):
        byte = lat[..., j].astype(np.int64)
        lo, hi = byte & 0xF, (byte >> 4) & 0xF
        out[..., 2 * j] = np.where(lo >= 8, lo - 16, lo)
        out[..., 2 * j + 1] = np.where(hi >= 8, hi - 16, hi)
    return out


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Integer codes [..., r] -> cache bytes (inverse of unpack_codes)."""
    codes = np.asarray(codes, dtype=np.int64)
    Q = qmax(bits)
    assert np.all(np.abs(codes) <= Q)
    if bits == 8:
        return (codes & 0xFF).astype(np.uint8)
    r = codes.shape[-1]
    out = np.empty(codes.shape[:-1] + (r // 2,), dtype=np.uint8)
    for j in range(r // 2):
        out[..., j] = ((codes[..., 2 * j] & 0xF) | ((codes[..., 2 * j + 1] & 0xF) << 4)).astype(np.uint8)
    return out


def dequantize(lat: np.ndarray, scale: np.ndarray, r: int, bits: int) -> np.ndarray:
    """Latent value = code * per-token scale (fp16 scale widened exactly)."""
    return unpack_codes(lat, r, bits).astype(np.float64) * np.asarray(scale, np.float64)[..., None]


def quantize(c: np.ndarray, bits: int) -> Tuple[np.ndarray, np.ndarray]:
    """Symmetric per-row quantiser of the latent cache (W8A8 / W8A4, de §2.C).

    scale = fp16(max|c| / Q); code = clip(round_half_even(c / scale), -Q, Q);
    a row with max|c| = 0 gets scale 0 and all-zero codes.  The division and
    the rounding decisions are taken in float32 (c is rounded to float32 first)
    so that they are the same decisions the kernel takes.
    Returns (codes int64 [..., r], scale float16 [...])."""
    Q = qmax(bits)
    c32 = np.asarray(c, dtype=np.float64).astype(np.float32)
    amax = np.max(np.abs(c32), axis=-1)
    scale = (amax / np.float32(Q)).astype(np.float16)
    s32 = scale.astype(np.float32)[..., None]
    safe = np.where(s32 > 0, s32, np.float32(1.0))
    v = np.where(s32 > 0, c32 / safe, np.float32(0.0)).astype(np.float32)
    codes = np.clip(np.rint(v), -Q, Q).astype(np.int64)
    return codes, scale


# ----------------------------------------------------------------------------- attention
def softmax(s: np.ndarray) -> np.ndarray:
    """p_l = exp(s_l - max s) / sum_k exp(s_k - max s)."""
    m = np.max(s)
    e = np.exp(s - m)
    return e / np.sum(e)


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, softmax_scale: float
              ) -> Tuple[np.ndarray, np.ndarray]:
    """Single-query attention out = softmax(q.K^T * softmax_scale) . V.
    Returns (out [Hd], p [L]).  An empty key set gives out = 0."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], np.float64), np.zeros(0, np.float64)
    s = (K @ q) * softmax_scale
    p = softmax(s)
    return p @ V, p


def default_scale(Hd: int, softmax_scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(Hd) if not softmax_scale else float(softmax_scale)


def wsvd_decode_head(q: np.ndarray, lat_k, scale_k, lat_v, scale_v, Bk_h, Bv_h, n: int,
                     r: int, bits: int, softmax_scale: Optional[float] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """One (b, h) of the decode step over the first n cached tokens.

    lat_K = code_K * s_K, K = lat_K . B_Kh (n x Hd), likewise V; then plain
    attention (ja §2.4 / de §2.D: q.K^T, softmax, V product).  Rows >= n are
    never read."""
    Hd = Bk_h.shape[1]
    latK = dequantize(lat_k[:n], scale_k[:n], r, bits)
    latV = dequantize(lat_v[:n], scale_v[:n], r, bits)
    K = latK @ np.asarray(Bk_h, np.float64)
    V = latV @ np.asarray(Bv_h, np.float64)
    return attention(np.asarray(q, np.float64), K, V, default_scale(Hd, softmax_scale))


def wsvd_decode(q, lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r: int, bits: int,
                softmax_scale: Optional[float] = None) -> np.ndarray:
    """Decode step over a per-head low-rank cache: out [B][H][Hd] float64.

    q [B][H][Hd]; lat_* [B][H][L_cap][r*bits/8]; scale_* [B][H][L_cap];
    Bk, Bv [H][r][Hd]; seq_lens [B] with 0 <= len_b <= L_cap."""
    B, H, Hd = q.shape
    out = np.zeros((B, H, Hd), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            out[b, h], _ = wsvd_decode_head(q[b, h], lat_k[b, h], scale_k[b, h], lat_v[b, h],
                                            scale_v[b, h], Bk[h], Bv[h], n, r, bits, softmax_scale)
    return out


def wsvd_decode_gqa(q, lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r: int, bits: int,
                    softmax_scale: Optional[float] = None) -> np.ndarray:
    """Grouped-query decode over a per-head low-rank cache: out [B][Hq][Hd].

    Hq query heads share Hkv latent heads (Hq = G * Hkv): query head g reads
    latent head g // G with that head's factors, i.e. consecutive query heads
    form a group, as in grouped-query attention.  q [B][Hq][Hd]; lat_*,
    scale_* over Hkv heads; Bk, Bv [Hkv][r][Hd].  The pages describe one
    query per latent head; this is the grouped reading of the same decode
    (each query head is the plain decode of ja §2.4 / de §2.D over its
    group's latent)."""
    B, Hq, Hd = q.shape
    Hkv = lat_k.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of latent heads")
    G = Hq // Hkv
    out = np.zeros((B, Hq, Hd), np.float64)
    for b in range(B):
        n = int(seq_lens[b])
        for g in range(Hq):
            j = g // G
            out[b, g], _ = wsvd_decode_head(q[b, g], lat_k[b, j], scale_k[b, j], lat_v[b, j], scale_v[b, j],
                                            Bk[j], Bv[j], n, r, bits, softmax_scale)
    return out


def wsvd_decode_multi(q, lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r: int, bits: int,
                      softmax_scale: Optional[float] = None) -> np.ndarray:
    """Decode of Tq new tokens per sequence at once (a speculative or chunked
    decode step): out [B][Tq][Hq][Hd].

    q [B][Tq][Hq][Hd]; the Tq tokens are the last Tq cached rows of each
    sequence, so query t of sequence b sees rows [0, seq_lens[b] - Tq + 1 + t)
    (causal inside the block, everything before it).  Latent heads may be
    grouped as in wsvd_decode_gqa.  A query that sees no row gets 0."""
    B, Tq, Hq, Hd = q.shape
    out = np.zeros((B, Tq, Hq, Hd), np.float64)
    for t in range(Tq):
        n_t = np.maximum(np.asarray(seq_lens, np.int64) - Tq + 1 + t, 0)
        out[:, t] = wsvd_decode_gqa(q[:, t], lat_k, scale_k, lat_v, scale_v, Bk, Bv, n_t, r, bits, softmax_scale)
    return out


def dense_decode(q, K, V, seq_lens, softmax_scale: Optional[float] = None) -> np.ndarray:
    """Textbook decode over a dense fp16 KV cache: the flash-decoding baseline
    the pages compare against (de §4 "Ergebnisse").  K, V [B][H][L_cap][Hd]."""
    B, H, Hd = q.shape
    out = np.zeros((B, H, Hd), np.float64)
    sc = default_scale(Hd, softmax_scale)
    for b in range(B):
        n = int(seq_lens[b])
        for h in range(H):
            out[b, h], _ = attention(np.asarray(q[b, h], np.float64), np.asarray(K[b, h, :n], np.float64),
                                     np.asarray(V[b, h, :n], np.float64), sc)
    return out


def shared_latent_decode(q, lat_k, lat_v, Bk, Bv, seq_lens,
                         softmax_scale: Optional[float] = None) -> np.ndarray:
    """Conventional SVD decode: every head rebuilds its K and V from one latent
    shared by all heads, lat [B][L_cap][R], with per-head B [H][R][Hd]
    (the re-read of the shared latent the pages blame: ja §1, de §1)."""
    B, H, Hd = q.shape
    out = np.zeros((B, H, Hd), np.float64)
    sc = default_scale(Hd, softmax_scale)
    for b in range(B):
        n = int(seq_lens[b])
        LK = np.asarray(lat_k[b, :n], np.float64)
        LV = np.asarray(lat_v[b, :n], np.float64)
        for h in range(H):
            K = LK @ np.asarray(Bk[h], np.float64)
            V = LV @ np.asarray(Bv[h], np.float64)
            out[b, h], _ = attention(np.asarray(q[b, h], np.float64), K, V, sc)
    return out


# ----------------------------------------------------------------------------- rotation + append
def sylvester_hadamard(n: int) -> np.ndarray:
    """Unnormalised Hadamard matrix of order n (a power of two) in Sylvester's
    natural order: H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]]."""
    if n < 1 or n & (n - 1):
        raise ValueError("Hadamard order must be a power of two")
    Hm = np.ones((1, 1), np.float64)
    while Hm.shape[0] < n:
        Hm = np.block([[Hm, Hm], [Hm, -Hm]])
    return Hm


def block_hadamard_rotate(x: np.ndarray, block: int) -> np.ndarray:
    """x~ = x . blockdiag(H_block / sqrt(block)): the orthonormal rotation S1 of
    the activations (de §2.C: S1 is a Hadamard matrix), one block at a time."""
    x = np.asarray(x, np.float64)
    E = x.shape[-1]
    if E % block:
        raise ValueError("E must be a multiple of the Hadamard block")
    Hn = sylvester_hadamard(block) / math.sqrt(block)
    out = np.empty_like(x)
    for s in range(0, E, block):
        out[..., s:s + block] = x[..., s:s + block] @ Hn
    return out


def latent_project(x, A_k, A_v, block: int) -> Tuple[np.ndarray, np.ndarray]:
    """c_K[b,h] = x~[b] . A_Kh and c_V[b,h] = x~[b] . A_Vh (A_h in R^{E x r},
    ar §2.a), x~ the Hadamard-rotated activation.  Returns [B][H][r] twice."""
    xt = block_hadamard_rotate(x, block)
    ck = np.einsum("be,her->bhr", xt, np.asarray(A_k, np.float64))
    cv = np.einsum("be,her->bhr", xt, np.asarray(A_v, np.float64))
    return ck, cv


def latent_append(x, A_k, A_v, seq_lens, lat_k, scale_k, lat_v, scale_v, r: int, bits: int,
                  block: int):
    """Write one new token per sequence into the latent cache.

    For each b with 0 <= seq_lens[b] < L_cap: rotate, project through A_Kh and
    A_Vh, quantise each (b, h, K|V) row and store it at row seq_lens[b], then
    seq_lens[b] += 1.  A sequence whose cache is full is left untouched and
    flagged.  Returns (lat_k, scale_k, lat_v, scale_v, seq_lens, err_rows,
    ck, cv) as new arrays; err_rows[b] is True where the row was refused."""
    ck, cv = latent_project(x, A_k, A_v, block)
    lat_k, lat_v = lat_k.copy(), lat_v.copy()
    scale_k, scale_v = scale_k.copy(), scale_v.copy()
    lens = np.asarray(seq_lens, np.int64).copy()
    B, H = ck.shape[:2]
    L_cap = lat_k.shape[2]
    err = np.zeros(B, bool)
    for b in range(B):
        pos = int(lens[b])
        if pos < 0 or pos >= L_cap:
            err[b] = True
            continue
        for h in range(H):
            codes, s = quantize(ck[b, h], bits)
            lat_k[b, h, pos] = pack_codes(codes, bits)
            scale_k[b, h, pos] = s
            codes, s = quantize(cv[b, h], bits)
            lat_v[b, h, pos] = pack_codes(codes, bits)
            scale_v[b, h, pos] = s
        lens[b] = pos + 1
    return lat_k, scale_k, lat_v, scale_v, lens.astype(np.int32), err, ck, cv


def latent_prefill(x, A_k, A_v, seq_lens, lat_k, scale_k, lat_v, scale_v, r: int, bits: int, block: int):
    """Write a block of T new tokens per sequence into the latent cache (the
    prompt's tokens, e.g. the image tokens of a vision-language prompt, in one
    call instead of T single-token appends).

    x [B][T][E].  Each token is rotated, projected and quantised exactly as by
    latent_append (the per-head projection of German §2.A after the rotation
    S1 and the W8A8 / W8A4 quantiser of German §2.C): token t of sequence b
    goes to row seq_lens[b] + t, then seq_lens[b] += T.  The pages describe
    the cache and its per-token quantiser, not a block interface; the block
    write is read as the same rows that T successive appends would write.
    A sequence whose block does not fit (seq_lens[b] < 0 or
    seq_lens[b] + T > L_cap) is left untouched and flagged.
    Returns (lat_k, scale_k, lat_v, scale_v, seq_lens, err_rows, ck, cv) with
    ck, cv [B][T][H][r] float64."""
    x = np.asarray(x, np.float64)
    B, T, E = x.shape
    xt = block_hadamard_rotate(x, block)
    H = np.shape(A_k)[0]
    ck = np.stack([xt @ np.asarray(A_k[h], np.float64) for h in range(H)], axis=2)  # [B][T][H][r]
    cv = np.stack([xt @ np.asarray(A_v[h], np.float64) for h in range(H)], axis=2)
    lat_k, lat_v = lat_k.copy(), lat_v.copy()
    scale_k, scale_v = scale_k.copy(), scale_v.copy()
    lens = np.asarray(seq_lens, np.int64).copy()
    L_cap = lat_k.shape[2]
    err = np.zeros(B, bool)
    for b in range(B):
        pos = int(lens[b])
        if pos < 0 or pos + T > L_cap:
            err[b] = True
            continue
        for t in range(T):
            for h in range(H):
                codes, s = quantize(ck[b, t, h], bits)
                lat_k[b, h, pos + t] = pack_codes(codes, bits)
                scale_k[b, h, pos + t] = s
                codes, s = quantize(cv[b, t, h], bits)
                lat_v[b, h, pos + t] = pack_codes(codes, bits)
                scale_v[b, h, pos + t] = s
        lens[b] = pos + T
    return lat_k, scale_k, lat_v, scale_v, lens.astype(np.int32), err, ck, cv


# ----------------------------------------------------------------------------- footprint
# ----------------------------------------------------------------------------- latent rotation S2
def fold_latent_rotation(A: np.ndarray, B: np.ndarray, S2: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Fold an orthogonal rotation S2 of each head's latent space into its
    factors: A' = A . S2 (A [H][E][r]) and B' = S2^T . B (B [H][r][Hd]),
    S2 [H][r][r] orthogonal (float64).

    The pages introduce orthogonal transforms S1 (the Hadamard rotation of the
    activations) and S2, learned jointly with A and B to smooth what is
    quantised (de §2.C "Outlier-Smoothing", ar §2.c).  Reading taken: S2 acts
    on the r-dimensional latent of each head (one for K, one for V), so the
    cache holds rotated latents c . S2 and, since S2 . S2^T = I, folding it
    into A and B leaves c . B unchanged."""
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    S2 = np.asarray(S2, np.float64)
    return np.einsum("her,hrs->hes", A, S2), np.einsum("hrs,hrd->hsd", S2, B)


# ----------------------------------------------------------------------------- int8 weights
def dequantize_weights(wq: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Int8 weight matrices wq [H][K][N] with one scale per output column,
    scale [H][N]: W[h][k][n] = wq[h][k][n] * scale[h][n] (float64).

    The "W8" of the method's W8A8 / W8A4 configurations (de §2.C): the low-rank
    factors A_h (E x r, output columns r) and B_h (r x Hd, output columns Hd)
    stored as 8-bit weights.  The pages fix no scale granularity; one scale per
    output column is the reading taken here."""
    return np.asarray(wq, np.float64) * np.asarray(scale, np.float64)[:, None, :]


def wsvd_cache_bytes(B: int, H: int, L_cap: int, r: int, bits: int) -> int:
    """Per-head latent cache: K and V codes (L x r each, bits per code) plus one
    fp16 scale per token per head for each (ar §2.a: footprint L x r per head)."""
    return B * H * L_cap * (2 * r * bits // 8 + 2 * 2)


def shared_cache_bytes(B: int, L_cap: int, R: int) -> int:
    """Shared fp16 latent of a conventional SVD: L x R for K and for V."""
    return B * L_cap * 2 * R * 2


def dense_cache_bytes(B: int, H: int, L_cap: int, Hd: int) -> int:
    """Dense fp16 K and V: L x Hd per head each."""
    return B * H * L_cap * 2 * Hd * 2
