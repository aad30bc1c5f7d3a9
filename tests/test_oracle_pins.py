"""Pins for the float64 oracle: each check ties the oracle to something other
than itself (brute force in exact arithmetic, closed forms, library routines,
hand-derived fixtures under tests/golden/, invariants of attention)."""
import math
import os
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


# ----------------------------------------------------------------------------- storage formats
def test_int4_layout_golden():
    for tok in _golden_lines("int4_nibbles.txt"):
        byte, even, odd = int(tok[0], 16), int(tok[1]), int(tok[2])
        got = O.unpack_codes(np.array([[byte]], np.uint8), 2, 4)[0]
        assert list(got) == [even, odd], tok


def test_int4_all_bytes_closed_form():
    # Two's complement nibble value: n - 16 if n >= 8; low nibble is the even element.
    allb = np.arange(256, dtype=np.uint8)[:, None]
    got = O.unpack_codes(allb, 2, 4)
    for b in range(256):
        lo, hi = b % 16, b // 16
        assert got[b, 0] == (lo - 16 if lo >= 8 else lo)
        assert got[b, 1] == (hi - 16 if hi >= 8 else hi)


def test_int8_all_bytes_closed_form():
    allb = np.arange(256, dtype=np.uint8)[:, None]
    got = O.unpack_codes(allb, 1, 8)[:, 0]
    assert all(got[b] == (b - 256 if b >= 128 else b) for b in range(256))


@pytest.mark.parametrize("bits", [8, 4])
def test_pack_roundtrip(bits):
    Q = O.qmax(bits)
    rng = np.random.default_rng(1)
    codes = rng.integers(-Q, Q + 1, size=(5, 7, 32))
    assert np.array_equal(O.unpack_codes(O.pack_codes(codes, bits), 32, bits), codes)
    # The generator's storage step writes the same layout.
    assert np.array_equal(W.store_codes(codes, bits), O.pack_codes(codes, bits))


# ----------------------------------------------------------------------------- quantiser
@pytest.mark.parametrize("bits", [8, 4])
def test_quantize_exact_dyadic_bruteforce(bits):
    """Rows built so that every value, the scale and every ratio are exact in
    float32: then the nearest code is decided exactly, and an exhaustive search
    over all 2Q+1 codes (ties to the even code) must agree."""
    Q = O.qmax(bits)
    rng = np.random.default_rng(7)
    for e in range(-6, 4):
        scale = 2.0 ** e
        m = rng.integers(-8 * Q, 8 * Q + 1, size=(40, 16))  # v = m/8 in [-Q, Q]
        m[:, 0] = 8 * Q  # amax = Q * scale exactly
        c = m / 8.0 * scale
        codes, s = O.quantize(c, bits)
        assert np.all(s.astype(np.float64) == scale)
        for i in range(m.shape[0]):
            for j in range(m.shape[1]):
                v = Fraction(int(m[i, j]), 8)
                best = min(range(-Q, Q + 1), key=lambda k: (abs(v - k), k % 2))
                assert codes[i, j] == best, (v, codes[i, j], best)


def test_quantize_ties_to_even_and_clamp():
    # scale = 1 (amax = Q); v = 2.5 -> 2, 3.5 -> 4, -2.5 -> -2, -0.5 -> 0
    c = np.array([[127.0, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5]])
    codes, s = O.quantize(c, 8)
    assert float(s[0]) == 1.0
    assert list(codes[0]) == [127, 2, 4, -2, 0, 0, 2]
    # amax/Q rounds down in fp16, so amax/scale > Q: the code is clamped to Q.
    amax = 7.0 * (1.0 + 2.0 ** -12)  # fp16(amax/7) = 1.0
    codes, s = O.quantize(np.array([[amax, -amax, 1.0]]), 4)
    assert float(s[0]) == 1.0
    assert list(codes[0]) == [7, -7, 1]


def test_quantize_zero_row():
    codes, s = O.quantize(np.zeros((3, 32)), 8)
    assert np.all(codes == 0) and np.all(s == 0)


@pytest.mark.parametrize("bits", [8, 4])
def test_quantize_random_rows_properties(bits):
    """scale = fp16(float32(amax)/Q) via Python's struct half-precision packing;
    codes within half a step of c / scale unless clamped; argmax hits +-Q."""
    import struct
    Q = O.qmax(bits)
    rng = np.random.default_rng(3)
    c = rng.standard_t(3, size=(200, 32)) * rng.choice([1e-3, 1.0, 30.0], size=(200, 1))
    codes, s = O.quantize(c, bits)
    c32 = c.astype(np.float32)
    for i in range(c.shape[0]):
        amax = float(np.max(np.abs(c32[i])))
        ratio = float(np.float32(amax) / np.float32(Q))
        want = struct.unpack("<e", struct.pack("<e", ratio))[0]
        assert float(s[i]) == want
        sc = float(s[i])
        v = c32[i].astype(np.float64) / sc
        assert np.all(np.abs(codes[i] - v)[np.abs(v) <= Q] <= 0.5 + 1e-6)
        j = int(np.argmax(np.abs(c32[i])))
        assert abs(codes[i, j]) == Q


# ----------------------------------------------------------------------------- Hadamard S1
def test_hadamard_golden_order8():
    want = np.array([[int(t) for t in row] for row in _golden_lines("hadamard8.txt")], np.float64)
    assert np.array_equal(O.sylvester_hadamard(8), want)


@pytest.mark.parametrize("n", [1, 2, 16, 128])
def test_hadamard_library_and_walsh_closed_form(n):
    Hm = O.sylvester_hadamard(n)
    assert np.array_equal(Hm, scipy.linalg.hadamard(n).astype(np.float64))
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pop = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    assert np.array_equal(Hm, (-1.0) ** pop)
    assert np.allclose(Hm @ Hm.T, n * np.eye(n))


def test_block_rotation_orthonormal_and_blockwise():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 512))
    xt = O.block_hadamard_rotate(x, 128)
    assert np.allclose(np.linalg.norm(xt, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    # A unit vector in block 2 lands on row i of H/sqrt(128) inside block 2 only.
    e = np.zeros((1, 512))
    e[0, 256 + 5] = 1.0
    t = O.block_hadamard_rotate(e, 128)[0]
    ref = scipy.linalg.hadamard(128)[5] / math.sqrt(128)
    assert np.allclose(t[256:384], ref, atol=1e-15) and np.all(t[:256] == 0) and np.all(t[384:] == 0)


def test_projection_undoes_rotation():
    """With A_h = blockdiag(H/sqrt(n))^T . A'_h the rotated projection equals x . A'_h:
    a wrong order or normalisation of the rotation breaks the identity."""
    rng = np.random.default_rng(4)
    E, Hh, r, blk = 256, 3, 8, 128
    x = rng.standard_normal((2, E))
    Ap = rng.standard_normal((Hh, E, r))
    Hn = scipy.linalg.hadamard(blk) / math.sqrt(blk)
    Rt = scipy.linalg.block_diag(*[Hn] * (E // blk))
    A = np.einsum("fe,her->hfr", Rt.T, Ap)  # A[h] = Rt^T @ Ap[h]
    ck, cv = O.latent_project(x, A, -A, blk)
    want = np.einsum("be,her->bhr", x, Ap)
    assert np.allclose(ck, want, atol=1e-12) and np.allclose(cv, -want, atol=1e-12)


# ----------------------------------------------------------------------------- decode: brute force
def _exact_decode_head(q, codes_k, sk, codes_v, sv, Bk, Bv, n, digits=50):
    """Exact rationals for the scores (all inputs are dyadic), mpmath for exp."""
    mpmath.mp.dps = digits
    r, Hd = Bk.shape
    Fq = [Fraction(float(v)) for v in q]
    K = [[sum(Fraction(int(codes_k[l][j])) * Fraction(float(sk[l])) * Fraction(float(Bk[j][d]))
              for j in range(r)) for d in range(Hd)] for l in range(n)]
    V = [[sum(Fraction(int(codes_v[l][j])) * Fraction(float(sv[l])) * Fraction(float(Bv[j][d]))
              for j in range(r)) for d in range(Hd)] for l in range(n)]
    raw = [sum(K[l][d] * Fq[d] for d in range(Hd)) for l in range(n)]
    scale = mpmath.mpf(1) / mpmath.sqrt(Hd)
    s = [mpmath.mpf(x.numerator) / x.denominator * scale for x in raw]
    m = max(s)
    e = [mpmath.exp(x - m) for x in s]
    Z = sum(e)
    out = [sum(e[l] / Z * (mpmath.mpf(V[l][d].numerator) / V[l][d].denominator) for l in range(n))
           for d in range(Hd)]
    return np.array([float(v) for v in out]), np.array([float(x / Z) for x in e])


@pytest.mark.parametrize("bits,r,Hd,n", [(8, 2, 4, 1), (8, 3, 5, 4), (4, 4, 3, 8), (8, 6, 8, 7)])
def test_decode_matches_exact_bruteforce(bits, r, Hd, n):
    rng = np.random.default_rng(100 + n)
    Q = O.qmax(bits)
    ck = rng.integers(-Q, Q + 1, size=(n, r))
    cv = rng.integers(-Q, Q + 1, size=(n, r))
    sk = rng.uniform(0.01, 0.1, n).astype(np.float16)
    sv = rng.uniform(0.01, 0.1, n).astype(np.float16)
    Bk = (rng.standard_normal((r, Hd)) / math.sqrt(r)).astype(np.float16)
    Bv = (rng.standard_normal((r, Hd)) / math.sqrt(r)).astype(np.float16)
    q = rng.standard_normal(Hd).astype(np.float16)
    pad = 3  # rows beyond n hold garbage the oracle must not read
    lk = O.pack_codes(np.vstack([ck, np.full((pad, r), Q)]), bits)
    lv = O.pack_codes(np.vstack([cv, np.full((pad, r), -Q)]), bits)
    sk2 = np.concatenate([sk, np.full(pad, np.float16(np.nan))])
    sv2 = np.concatenate([sv, np.full(pad, np.float16(np.inf))])
    got, p = O.wsvd_decode_head(q, lk, sk2, lv, sv2, Bk, Bv, n, r, bits)
    want, pw = _exact_decode_head(q, ck, sk, cv, sv, Bk, Bv, n)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
    assert np.allclose(p, pw, rtol=1e-12, atol=1e-300)


def test_two_token_golden():
    rows = {t[0]: np.array([float(v) for v in t[1:]]) for t in _golden_lines("two_token_logistic.txt")}
    ck = np.array([[0, 0, 0, 0], [2, 0, 0, 0]])
    cv = np.array([[1, 0, 0, 0], [0, 1, 0, 0]])
    s = np.ones(2, np.float16)
    I4 = np.eye(4, dtype=np.float16)
    lk, lv = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    out, _ = O.wsvd_decode_head(np.array([1, 0, 0, 0], np.float16), lk, s, lv, s, I4, I4, 2, 4, 8)
    assert np.allclose(out, rows["out"], rtol=1e-15, atol=1e-16)
    out0, _ = O.wsvd_decode_head(np.zeros(4, np.float16), lk, s, lv, s, I4, I4, 2, 4, 8)
    assert np.allclose(out0, rows["out_q0"], rtol=0, atol=1e-16)


# ----------------------------------------------------------------------------- decode: special cases
def _sdpa(q, K, V, scale):
    """torch's scaled_dot_product_attention in float64 for one query."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, None, None, :]
    Kt = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    Vt = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)[0, 0, 0].numpy()


@pytest.mark.parametrize("bits", [8, 4])
def test_identity_factor_reduces_to_standard_attention(bits):
    """r = Hd, B = I: the latents are K and V themselves, and the oracle must be
    standard attention over the dequantised K, V (torch's SDPA as the reference)."""
    rng = np.random.default_rng(11)
    B, H, Hd, L = 2, 3, 16, 37
    Q = O.qmax(bits)
    lens = np.array([37, 5])
    ck = rng.integers(-Q, Q + 1, size=(B, H, L, Hd))
    cv = rng.integers(-Q, Q + 1, size=(B, H, L, Hd))
    sk = rng.uniform(0.005, 0.05, (B, H, L)).astype(np.float16)
    sv = rng.uniform(0.005, 0.05, (B, H, L)).astype(np.float16)
    q = rng.standard_normal((B, H, Hd)).astype(np.float16)
    I = np.broadcast_to(np.eye(Hd, dtype=np.float16), (H, Hd, Hd))
    out = O.wsvd_decode(q, O.pack_codes(ck, bits), sk, O.pack_codes(cv, bits), sv, I, I, lens, Hd, bits)
    for b in range(B):
        n = lens[b]
        for h in range(H):
            K = ck[b, h, :n] * sk[b, h, :n, None].astype(np.float64)
            V = cv[b, h, :n] * sv[b, h, :n, None].astype(np.float64)
            ref = _sdpa(q[b, h], K, V, 1.0 / math.sqrt(Hd))
            assert np.allclose(out[b, h], ref, rtol=1e-12, atol=1e-14)


def _random_head(rng, n, r=4, Hd=8, bits=8):
    Q = O.qmax(bits)
    ck = rng.integers(-Q, Q + 1, size=(n, r))
    cv = rng.integers(-Q, Q + 1, size=(n, r))
    sk = rng.uniform(0.01, 0.1, n).astype(np.float16)
    sv = rng.uniform(0.01, 0.1, n).astype(np.float16)
    Bk = rng.standard_normal((r, Hd)).astype(np.float16)
    Bv = rng.standard_normal((r, Hd)).astype(np.float16)
    q = rng.standard_normal(Hd).astype(np.float16)
    return q, ck, sk, cv, sv, Bk, Bv


def test_identical_keys_give_mean_of_values():
    rng = np.random.default_rng(5)
    q, ck, sk, cv, sv, Bk, Bv = _random_head(rng, 9)
    ck[:] = ck[0]
    sk[:] = sk[0]
    out, p = O.wsvd_decode_head(q, O.pack_codes(ck, 8), sk, O.pack_codes(cv, 8), sv, Bk, Bv, 9, 4, 8)
    V = (cv * sv[:, None].astype(np.float64)) @ Bv.astype(np.float64)
    assert np.allclose(out, V.mean(axis=0), rtol=1e-13, atol=1e-14)
    assert np.allclose(p, 1.0 / 9, rtol=1e-14)


def test_zero_query_gives_mean_and_single_token_gives_v0():
    rng = np.random.default_rng(6)
    q, ck, sk, cv, sv, Bk, Bv = _random_head(rng, 6)
    lk, lv = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    V = (cv * sv[:, None].astype(np.float64)) @ Bv.astype(np.float64)
    out, _ = O.wsvd_decode_head(np.zeros_like(q), lk, sk, lv, sv, Bk, Bv, 6, 4, 8)
    assert np.allclose(out, V.mean(axis=0), rtol=1e-13, atol=1e-14)
    out1, p1 = O.wsvd_decode_head(q, lk, sk, lv, sv, Bk, Bv, 1, 4, 8)
    assert np.array_equal(p1, [1.0]) and np.allclose(out1, V[0], rtol=1e-15, atol=0)


def test_weights_sum_to_one_and_permutation_invariance():
    rng = np.random.default_rng(8)
    q, ck, sk, cv, sv, Bk, Bv = _random_head(rng, 50, r=8, Hd=16)
    lk, lv = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    out, p = O.wsvd_decode_head(q, lk, sk, lv, sv, Bk, Bv, 50, 8, 8)
    assert abs(p.sum() - 1.0) < 1e-14 and np.all(p > 0)
    perm = rng.permutation(50)
    out2, p2 = O.wsvd_decode_head(q, lk[perm], sk[perm], lv[perm], sv[perm], Bk, Bv, 50, 8, 8)
    assert np.allclose(out, out2, rtol=1e-13, atol=1e-14) and np.allclose(p[perm], p2, rtol=1e-13)


def test_empty_sequence_gives_zero():
    rng = np.random.default_rng(9)
    q, ck, sk, cv, sv, Bk, Bv = _random_head(rng, 4)
    out, p = O.wsvd_decode_head(q, O.pack_codes(ck, 8), sk, O.pack_codes(cv, 8), sv, Bk, Bv, 0, 4, 8)
    assert np.all(out == 0) and p.size == 0


def test_dense_oracle_matches_sdpa():
    rng = np.random.default_rng(12)
    B, H, L, Hd = 2, 2, 30, 8
    lens = np.array([30, 13])
    K = rng.standard_normal((B, H, L, Hd)).astype(np.float16)
    V = rng.standard_normal((B, H, L, Hd)).astype(np.float16)
    q = rng.standard_normal((B, H, Hd)).astype(np.float16)
    out = O.dense_decode(q, K, V, lens)
    for b in range(B):
        for h in range(H):
            n = lens[b]
            ref = _sdpa(q[b, h], K[b, h, :n].astype(np.float64), V[b, h, :n].astype(np.float64),
                        1 / math.sqrt(Hd))
            assert np.allclose(out[b, h], ref, rtol=1e-12, atol=1e-14)


def test_shared_latent_with_selector_factors_equals_dense():
    """A shared latent that is the concatenation of every head's K (R = H*Hd) and
    per-head B that select head h's block must reproduce dense attention."""
    rng = np.random.default_rng(13)
    B, H, L, Hd = 2, 3, 20, 4
    R = H * Hd
    lens = np.array([20, 7])
    K = rng.standard_normal((B, H, L, Hd)).astype(np.float16)
    V = rng.standard_normal((B, H, L, Hd)).astype(np.float16)
    q = rng.standard_normal((B, H, Hd)).astype(np.float16)
    latk = np.concatenate([K[:, h] for h in range(H)], axis=-1)  # [B][L][R]
    latv = np.concatenate([V[:, h] for h in range(H)], axis=-1)
    sel = np.zeros((H, R, Hd), np.float16)
    for h in range(H):
        sel[h, h * Hd:(h + 1) * Hd] = np.eye(Hd)
    a = O.shared_latent_decode(q, latk, latv, sel, sel, lens)
    d = O.dense_decode(q, K, V, lens)
    assert np.allclose(a, d, rtol=1e-13, atol=1e-14)


def test_wsvd_equals_shared_when_each_head_owns_its_block():
    """Per-head latents embedded in disjoint blocks of a shared latent, with B
    zero outside the head's block, give the same decode: the two paths compute
    the same attention and differ only in what each head reads."""
    rng = np.random.default_rng(14)
    B, H, L, Hd, r = 1, 2, 11, 8, 4
    lens = np.array([11])
    ck = rng.integers(-127, 128, size=(B, H, L, r))
    cv = rng.integers(-127, 128, size=(B, H, L, r))
    sk = rng.uniform(0.01, 0.05, (B, H, L)).astype(np.float16)
    sv = rng.uniform(0.01, 0.05, (B, H, L)).astype(np.float16)
    Bk = rng.standard_normal((H, r, Hd)).astype(np.float16)
    Bv = rng.standard_normal((H, r, Hd)).astype(np.float16)
    q = rng.standard_normal((B, H, Hd)).astype(np.float16)
    w = O.wsvd_decode(q, O.pack_codes(ck, 8), sk, O.pack_codes(cv, 8), sv, Bk, Bv, lens, r, 8)
    latk = np.concatenate([ck[:, h] * sk[:, h, :, None].astype(np.float64) for h in range(H)], -1)
    latv = np.concatenate([cv[:, h] * sv[:, h, :, None].astype(np.float64) for h in range(H)], -1)
    BK = np.zeros((H, H * r, Hd))
    BV = np.zeros((H, H * r, Hd))
    for h in range(H):
        BK[h, h * r:(h + 1) * r] = Bk[h]
        BV[h, h * r:(h + 1) * r] = Bv[h]
    s = O.shared_latent_decode(q, latk, latv, BK, BV, lens)
    assert np.allclose(w, s, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- grouped and multi-token queries
def _gqa_case(seed, B=2, Hq=6, Hkv=2, Hd=8, r=4, L=11, bits=8):
    rng = np.random.default_rng(seed)
    Q = O.qmax(bits)
    ck = rng.integers(-Q, Q + 1, size=(B, Hkv, L, r))
    cv = rng.integers(-Q, Q + 1, size=(B, Hkv, L, r))
    sk = rng.uniform(0.01, 0.1, (B, Hkv, L)).astype(np.float16)
    sv = rng.uniform(0.01, 0.1, (B, Hkv, L)).astype(np.float16)
    Bk = (rng.standard_normal((Hkv, r, Hd)) / 2).astype(np.float16)
    Bv = (rng.standard_normal((Hkv, r, Hd)) / 2).astype(np.float16)
    return ck, cv, sk, sv, Bk, Bv, rng


def _rebuilt(codes, scale, Bm):
    """K or V of every (b, latent head) rebuilt with plain numpy: [B][Hkv][L][Hd]."""
    lat = codes.astype(np.float64) * scale.astype(np.float64)[..., None]
    return np.einsum("bjlr,jrd->bjld", lat, Bm.astype(np.float64))


@pytest.mark.parametrize("bits", [8, 4])
def test_gqa_matches_torch_grouped_sdpa(bits):
    """Query head g reads latent head g // G: torch's SDPA with enable_gqa (which
    groups consecutive query heads) on the rebuilt K, V is the reference; a
    strided grouping (g % Hkv) or a swapped factor fails it."""
    ck, cv, sk, sv, Bk, Bv, rng = _gqa_case(31, bits=bits)
    B, Hkv, L, r = ck.shape
    Hq, Hd = 6, Bk.shape[2]
    q = rng.standard_normal((B, Hq, Hd)).astype(np.float16)
    lens = np.array([L, 4])
    out = O.wsvd_decode_gqa(q, O.pack_codes(ck, bits), sk, O.pack_codes(cv, bits), sv, Bk, Bv, lens, r, bits)
    K, V = _rebuilt(ck, sk, Bk), _rebuilt(cv, sv, Bv)
    for b in range(B):
        n = lens[b]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b].astype(np.float64))[None, :, None, :], torch.from_numpy(K[b, :, :n])[None],
            torch.from_numpy(V[b, :, :n])[None], scale=1.0 / math.sqrt(Hd), enable_gqa=True)[0, :, 0].numpy()
        assert np.allclose(out[b], ref, rtol=1e-12, atol=1e-14)


def test_gqa_with_one_query_per_head_is_the_decode_and_expands_to_it():
    """G = 1 is wsvd_decode itself; G > 1 equals wsvd_decode on a cache whose
    latent heads and factors are each repeated G times."""
    ck, cv, sk, sv, Bk, Bv, rng = _gqa_case(32, Hq=2, Hkv=2)
    lk, lv = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    lens = np.array([11, 7])
    q2 = rng.standard_normal((2, 2, 8))
    assert np.array_equal(O.wsvd_decode_gqa(q2, lk, sk, lv, sv, Bk, Bv, lens, 4, 8),
                          O.wsvd_decode(q2, lk, sk, lv, sv, Bk, Bv, lens, 4, 8))
    q6 = rng.standard_normal((2, 6, 8))
    rep = lambda a, ax: np.repeat(a, 3, axis=ax)
    want = O.wsvd_decode(q6, rep(lk, 1), rep(sk, 1), rep(lv, 1), rep(sv, 1), rep(Bk, 0), rep(Bv, 0), lens, 4, 8)
    assert np.array_equal(O.wsvd_decode_gqa(q6, lk, sk, lv, sv, Bk, Bv, lens, 4, 8), want)


def test_multi_token_decode_is_causal_inside_the_block():
    """Tq new tokens at once: query t sees rows [0, len - Tq + 1 + t).  Checked
    against torch's SDPA with an explicit boolean mask built from that rule,
    and Tq = 1 against the single-token grouped decode."""
    ck, cv, sk, sv, Bk, Bv, rng = _gqa_case(33, L=13)
    B, Hkv, L, r = ck.shape
    Hq, Hd, Tq = 6, 8, 4
    lk, lv = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    lens = np.array([13, 9])
    q = rng.standard_normal((B, Tq, Hq, Hd))
    out = O.wsvd_decode_multi(q, lk, sk, lv, sv, Bk, Bv, lens, r, 8)
    K, V = _rebuilt(ck, sk, Bk), _rebuilt(cv, sv, Bv)
    for b in range(B):
        n = lens[b]
        mask = np.zeros((Tq, n), bool)
        for t in range(Tq):
            mask[t, :n - Tq + 1 + t] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b].transpose(1, 0, 2))[None], torch.from_numpy(K[b, :, :n])[None],
            torch.from_numpy(V[b, :, :n])[None], attn_mask=torch.from_numpy(mask), scale=1.0 / math.sqrt(Hd),
            enable_gqa=True)[0].numpy().transpose(1, 0, 2)
        assert np.allclose(out[b], ref, rtol=1e-12, atol=1e-14)
    one = O.wsvd_decode_multi(q[:, -1:], lk, sk, lv, sv, Bk, Bv, lens, r, 8)[:, 0]
    assert np.array_equal(one, O.wsvd_decode_gqa(q[:, -1], lk, sk, lv, sv, Bk, Bv, lens, r, 8))


# ----------------------------------------------------------------------------- append
def test_append_writes_one_row_and_advances():
    rng = np.random.default_rng(15)
    B, H, E, r, L_cap = 3, 2, 256, 8, 5
    x = rng.standard_normal((B, E))
    Ak = (rng.standard_normal((H, E, r)) / 16).astype(np.float16)
    Av = (rng.standard_normal((H, E, r)) / 16).astype(np.float16)
    lat = rng.integers(0, 256, size=(B, H, L_cap, r), dtype=np.uint8)
    sc = rng.uniform(0, 1, (B, H, L_cap)).astype(np.float16)
    lens = np.array([0, 3, 5], np.int32)  # the last sequence is full
    lk, sk, lv, sv, nl, err, ck, cv = O.latent_append(x, Ak, Av, lens, lat, sc, lat, sc, r, 8, 128)
    assert list(nl) == [1, 4, 5] and list(err) == [False, False, True]
    for b in range(B):
        for h in range(H):
            for l in range(L_cap):
                written = (b, l) in ((0, 0), (1, 3))
                if not written:
                    assert np.array_equal(lk[b, h, l], lat[b, h, l]) and sk[b, h, l] == sc[b, h, l]
                    assert np.array_equal(lv[b, h, l], lat[b, h, l]) and sv[b, h, l] == sc[b, h, l]
            if b < 2:
                pos = lens[b]
                codes, s = O.quantize(ck[b, h], 8)
                assert np.array_equal(O.unpack_codes(lk[b, h, pos], r, 8), codes) and sk[b, h, pos] == s
                # dequantised latent within half a step of the projection
                assert np.all(np.abs(codes * float(s) - ck[b, h]) <= float(s) / 2 * (1 + 1e-6) + 1e-12)


# ----------------------------------------------------------------------------- prefill (block of T tokens)
def _prefill_case(seed, B=3, T=4, H=2, E=256, r=8, L_cap=9, bits=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, T, E))
    Ak = (rng.standard_normal((H, E, r)) / 16).astype(np.float16)
    Av = (rng.standard_normal((H, E, r)) / 16).astype(np.float16)
    rb = r * bits // 8
    lat = rng.integers(0, 256, size=(B, H, L_cap, rb), dtype=np.uint8)
    sc = rng.uniform(0, 1, (B, H, L_cap)).astype(np.float16)
    return x, Ak, Av, lat, sc


@pytest.mark.parametrize("bits", [8, 4])
def test_prefill_equals_successive_appends(bits):
    """The block write is the rows that T single-token appends write, one after
    the other (and T = 1 is the append itself)."""
    r, T = 8, 4
    x, Ak, Av, lat, sc = _prefill_case(21, T=T, r=r, bits=bits)
    lens = np.array([0, 2, 5], np.int32)  # 5 + 4 = 9 = L_cap: fits exactly
    got = O.latent_prefill(x, Ak, Av, lens, lat, sc, lat, sc, r, bits, 128)
    state = [lat, sc, lat, sc, lens]
    for t in range(T):
        lk, sk, lv, sv, nl, err, _, _ = O.latent_append(x[:, t], Ak, Av, state[4], state[0], state[1], state[2],
                                                        state[3], r, bits, 128)
        assert not err.any()
        state = [lk, sk, lv, sv, nl]
    for g, s in zip(got[:5], state):
        assert np.array_equal(g, s)
    assert not got[5].any()
    one = O.latent_prefill(x[:, :1], Ak, Av, lens, lat, sc, lat, sc, r, bits, 128)
    app = O.latent_append(x[:, 0], Ak, Av, lens, lat, sc, lat, sc, r, bits, 128)
    for g, s in zip(one[:6], app[:6]):
        assert np.array_equal(g, s)


def test_prefill_projection_is_one_dense_matmul():
    """c[b,t,h] = (x[b,t] . blockdiag(H/sqrt(blk))) . A_h as one library matmul
    over all B*T rows: catches a transposed rotation, a swapped head index or a
    token mixed into another token's row."""
    x, Ak, Av, lat, sc = _prefill_case(22, B=2, T=5, H=3, E=256, r=8, L_cap=5)
    Hn = scipy.linalg.hadamard(128) / math.sqrt(128)
    Rt = scipy.linalg.block_diag(Hn, Hn)
    X = x.reshape(-1, 256) @ Rt
    _, _, _, _, _, _, ck, cv = O.latent_prefill(x, Ak, Av, np.zeros(2, np.int32), lat, sc, lat, sc, 8, 8, 128)
    for h in range(3):
        assert np.allclose(ck[:, :, h].reshape(-1, 8), X @ Ak[h].astype(np.float64), rtol=1e-12, atol=1e-12)
        assert np.allclose(cv[:, :, h].reshape(-1, 8), X @ Av[h].astype(np.float64), rtol=1e-12, atol=1e-12)


def test_prefill_capacity_boundary_and_empty_block():
    x, Ak, Av, lat, sc = _prefill_case(23, T=4, L_cap=9)
    lens = np.array([6, -1, 5], np.int32)  # 6 + 4 > 9 refused; negative refused; 5 + 4 = 9 fits
    lk, sk, lv, sv, nl, err, _, _ = O.latent_prefill(x, Ak, Av, lens, lat, sc, lat, sc, 8, 8, 128)
    assert list(err) == [True, True, False] and list(nl) == [6, -1, 9]
    for b in (0, 1):
        assert np.array_equal(lk[b], lat[b]) and np.array_equal(sk[b], sc[b])
        assert np.array_equal(lv[b], lat[b]) and np.array_equal(sv[b], sc[b])
    assert np.array_equal(lk[2, :, :5], lat[2, :, :5]) and not np.array_equal(lk[2, :, 5:], lat[2, :, 5:])
    e = O.latent_prefill(x[:, :0], Ak, Av, lens, lat, sc, lat, sc, 8, 8, 128)
    assert np.array_equal(e[0], lat) and np.array_equal(e[4], np.array([6, -1, 5], np.int32)) and e[5][1]


# ----------------------------------------------------------------------------- footprint
def test_footprint_against_pages_and_arrays():
    g = {t[0]: float(t[1]) for t in _golden_lines("footprint.txt")}
    B, H, L, Hd = 2, 32, 1600, 128
    r = Hd // 2
    w8 = O.wsvd_cache_bytes(B, H, L, r, 8) - B * H * L * 4  # without the fp16 scales
    assert w8 / O.dense_cache_bytes(B, H, L, Hd) == g["w8_r_half_hd_vs_fp16_noscale"]
    per_head_fp16 = lambda rr: L * rr * 2
    assert per_head_fp16(32) / per_head_fp16(512) == g["per_head_fp16_r32_vs_shared_R512"]
    assert per_head_fp16(32) / (L * 128 * 2) == g["per_head_fp16_r32_vs_dense_hd128"]
    # The byte counts equal the sizes of the arrays the cache is made of.
    w = W.PR1
    d = W.decode_inputs(w)
    nb = d.lat_k.nbytes + d.lat_v.nbytes + d.scale_k.nbytes + d.scale_v.nbytes
    assert nb == O.wsvd_cache_bytes(w.B, w.H, w.L_cap, w.r, w.bits)
    s = W.shared_inputs(W.CMP[2048].with_(B=1, L_cap=16, lens=16))
    assert s["lat_k"].nbytes + s["lat_v"].nbytes == O.shared_cache_bytes(1, 16, 512)


def test_dequantize_weights_scales_each_output_column():
    """Hand-computed: one scale per output column (last axis), shared by every
    row of the contraction axis; a per-row scale would give other numbers."""
    wq = np.array([[[1, -2], [3, 4]]], np.int8)         # [H=1][K=2][N=2]
    s = np.array([[0.5, 2.0]], np.float32)               # [H][N]
    got = O.dequantize_weights(wq, s)
    assert np.array_equal(got, np.array([[[0.5, -4.0], [1.5, 8.0]]]))
    # an int8 matrix with unit scales is the matrix itself
    rng = np.random.default_rng(0)
    q = rng.integers(-127, 128, size=(3, 5, 7)).astype(np.int8)
    assert np.array_equal(O.dequantize_weights(q, np.ones((3, 7), np.float32)), q.astype(np.float64))


def test_fold_latent_rotation_pins():
    """S2 = I leaves the factors unchanged; a hand-worked 2 x 2 rotation; and
    for a random orthogonal S2 the rebuilt keys c . B and the attention output
    over unquantised latents are unchanged (to float64 rounding), while the
    latents themselves do change."""
    rng = np.random.default_rng(3)
    A = rng.standard_normal((2, 8, 4))
    B = rng.standard_normal((2, 4, 6))
    I = np.broadcast_to(np.eye(4), (2, 4, 4))
    a2, b2 = O.fold_latent_rotation(A, B, I)
    assert np.array_equal(a2, A) and np.array_equal(b2, B)
    # a quarter turn in the latent plane: columns (x, y) -> (-y, x)
    R = np.array([[[0.0, 1.0], [-1.0, 0.0]]])
    a, b = O.fold_latent_rotation(np.array([[[1.0, 2.0]]]), np.array([[[3.0], [5.0]]]), R)
    assert np.array_equal(a, np.array([[[-2.0, 1.0]]])) and np.array_equal(b, np.array([[[-5.0], [3.0]]]))
    # invariance for a random orthogonal S2 (one per head)
    w = W.PR1
    S2 = W.latent_rotation(w, seed=1).astype(np.float64)
    assert np.allclose(np.einsum("hrs,hts->hrt", S2, S2), np.eye(w.r)[None], atol=1e-6)
    x = rng.standard_normal((3, 8))
    A = rng.standard_normal((w.H, 8, w.r))
    B = rng.standard_normal((w.H, w.r, w.Hd))
    A2, B2 = O.fold_latent_rotation(A, B, S2)
    c, c2 = np.einsum("le,her->hlr", x, A), np.einsum("le,her->hlr", x, A2)
    assert not np.allclose(c, c2)
    K, K2 = np.einsum("hlr,hrd->hld", c, B), np.einsum("hlr,hrd->hld", c2, B2)
    assert np.allclose(K, K2, rtol=1e-5, atol=1e-5)   # S2 is float32-orthogonal
    q = rng.standard_normal(w.Hd)
    for h in range(w.H):
        o1, _ = O.attention(q, K[h], K[h], 0.125)
        o2, _ = O.attention(q, K2[h], K2[h], 0.125)
        assert np.allclose(o1, o2, rtol=1e-5, atol=1e-5)
