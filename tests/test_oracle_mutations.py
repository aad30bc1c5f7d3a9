"""Plant plausible mistakes in the oracle (on the CPU, by monkeypatching) and
check that the pins catch every one of them."""
import math

import numpy as np
import pytest

import oracle as O
import oracle.wsvd_oracle as OW
import test_oracle_pins as P


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(OW, name, fn)
    monkeypatch.setattr(O, name, fn)


def _decode_head_variant(kind):
    def f(q, lat_k, scale_k, lat_v, scale_v, Bk_h, Bv_h, n, r, bits, softmax_scale=None):
        Hd = Bk_h.shape[1]
        latK = OW.dequantize(lat_k[:n], scale_k[:n], r, bits)
        latV = OW.dequantize(lat_v[:n], scale_v[:n], r, bits)
        if kind == "no_scale_K":
            latK = OW.unpack_codes(lat_k[:n], r, bits).astype(np.float64)
        K = latK @ np.asarray(Bk_h, np.float64)
        V = latV @ np.asarray((Bk_h if kind == "swap_B" else Bv_h), np.float64)
        sc = 1.0 if kind == "no_softmax_scale" else OW.default_scale(Hd, softmax_scale)
        if kind == "sign":
            sc = -sc
        out, p = OW.attention(np.asarray(q, np.float64), K, V, sc)
        if kind == "drop_last_token" and n > 1:
            out, p = OW.attention(np.asarray(q, np.float64), K[:-1], V[:-1], sc)
        return out, p
    return f



@pytest.mark.parametrize("kind", ["swap_B", "no_softmax_scale", "no_scale_K", "sign", "drop_last_token"])
def test_decode_mutants_are_caught(monkeypatch, kind):
    _patch(monkeypatch, "wsvd_decode_head", _decode_head_variant(kind))
    with pytest.raises(AssertionError):
        P.test_decode_matches_exact_bruteforce(8, 3, 5, 4)


def test_nibble_order_mutant_is_caught(monkeypatch):
    orig = OW.unpack_codes

    def swapped(lat, r, bits):
        c = orig(lat, r, bits)
        if bits == 4:
            c = c.reshape(c.shape[:-1] + (r // 2, 2))[..., ::-1].reshape(c.shape)
        return c
    _patch(monkeypatch, "unpack_codes", swapped)
    with pytest.raises(AssertionError):
        P.test_int4_layout_golden()


def test_round_half_away_mutant_is_caught(monkeypatch):
    def q_away(c, bits):
        Q = OW.qmax(bits)
        c32 = np.asarray(c, np.float64).astype(np.float32)
        amax = np.max(np.abs(c32), axis=-1)
        scale = (amax / np.float32(Q)).astype(np.float16)
        s32 = scale.astype(np.float32)[..., None]
        v = np.where(s32 > 0, c32 / np.where(s32 > 0, s32, 1), 0)
        codes = np.clip(np.sign(v) * np.floor(np.abs(v) + 0.5), -Q, Q).astype(np.int64)
        return codes, scale
    _patch(monkeypatch, "quantize", q_away)
    with pytest.raises(AssertionError):
        P.test_quantize_ties_to_even_and_clamp()


def test_scale_without_fp16_rounding_mutant_is_caught(monkeypatch):
    def q_f32(c, bits):
        Q = OW.qmax(bits)
        c32 = np.asarray(c, np.float64).astype(np.float32)
        amax = np.max(np.abs(c32), axis=-1)
        scale = amax / np.float32(Q)
        v = np.where(scale[..., None] > 0, c32 / np.where(scale[..., None] > 0, scale[..., None], 1), 0)
        return np.clip(np.rint(v), -Q, Q).astype(np.int64), scale
    _patch(monkeypatch, "quantize", q_f32)
    with pytest.raises(AssertionError):
        P.test_quantize_random_rows_properties(8)


def test_unnormalised_rotation_mutant_is_caught(monkeypatch):
    def rot(x, block):
        x = np.asarray(x, np.float64)
        Hn = OW.sylvester_hadamard(block)
        out = np.empty_like(x)
        for s in range(0, x.shape[-1], block):
            out[..., s:s + block] = x[..., s:s + block] @ Hn
        return out
    _patch(monkeypatch, "block_hadamard_rotate", rot)
    with pytest.raises(AssertionError):
        P.test_projection_undoes_rotation()


def test_reversed_block_order_mutant_is_caught(monkeypatch):
    def rot(x, block):
        x = np.asarray(x, np.float64)
        Hn = OW.sylvester_hadamard(block) / math.sqrt(block)
        out = np.empty_like(x)
        E = x.shape[-1]
        for s in range(0, E, block):
            d = E - block - s  # writes block k into block (n-1-k)
            out[..., d:d + block] = x[..., s:s + block] @ Hn
        return out
    _patch(monkeypatch, "block_hadamard_rotate", rot)
    with pytest.raises(AssertionError):
        P.test_block_rotation_orthonormal_and_blockwise()


def test_shared_path_wrong_head_mutant_is_caught(monkeypatch):
    orig = OW.shared_latent_decode

    def wrong(q, lat_k, lat_v, Bk, Bv, seq_lens, softmax_scale=None):
        return orig(q, lat_k, lat_v, Bk[::-1], Bv, seq_lens, softmax_scale)
    _patch(monkeypatch, "shared_latent_decode", wrong)
    with pytest.raises(AssertionError):
        P.test_shared_latent_with_selector_factors_equals_dense()


@pytest.mark.parametrize("kind", ["B_not_transposed", "A_transposed_rotation", "dequant_per_row"])
def test_rotation_and_weight_mutants_are_caught(monkeypatch, kind):
    """Folding S2 (not S2^T) into B, rotating A by S2^T, or scaling int8 weights
    per row instead of per output column: the pins must fail."""
    if kind == "dequant_per_row":
        _patch(monkeypatch, "dequantize_weights",
               lambda wq, s: np.asarray(wq, np.float64) * np.asarray(s, np.float64)[:, :, None]
               if np.shape(s)[1] == np.shape(wq)[1] else np.asarray(wq, np.float64) * 0.0)
        with pytest.raises(AssertionError):
            P.test_dequantize_weights_scales_each_output_column()
        return

    def fold(A, B, S2):
        A = np.asarray(A, np.float64)
        B = np.asarray(B, np.float64)
        S2 = np.asarray(S2, np.float64)
        if kind == "B_not_transposed":
            return np.einsum("her,hrs->hes", A, S2), np.einsum("hsr,hrd->hsd", S2, B)
        return np.einsum("her,hsr->hes", A, S2), np.einsum("hrs,hrd->hsd", S2, B)
    _patch(monkeypatch, "fold_latent_rotation", fold)
    with pytest.raises(AssertionError):
        P.test_fold_latent_rotation_pins()


def _prefill_variant(kind):
    orig = OW.latent_prefill

    def f(x, A_k, A_v, seq_lens, lat_k, scale_k, lat_v, scale_v, r, bits, block):
        x = np.asarray(x, np.float64)
        if kind == "batch_rows_swapped" and x.shape[0] > 1:
            x = x[::-1]
        if kind == "tokens_reversed":
            x = x[:, ::-1]
        lens = np.asarray(seq_lens, np.int64)
        if kind == "accept_overflow":  # refuses only a full cache, clips the block at L_cap
            L_cap, T = lat_k.shape[2], x.shape[1]
            res = list(orig(x, A_k, A_v, lens, lat_k, scale_k, lat_v, scale_v, r, bits, block))
            res[:5] = [lat_k.copy(), scale_k.copy(), lat_v.copy(), scale_v.copy(), lens.astype(np.int32)]
            res[5] = np.ones(x.shape[0], bool)
            for b in range(x.shape[0]):
                pos = int(lens[b])
                if 0 <= pos < L_cap:
                    n = min(T, L_cap - pos)
                    one = orig(x[b:b + 1, :n], A_k, A_v, lens[b:b + 1], lat_k[b:b + 1], scale_k[b:b + 1],
                               lat_v[b:b + 1], scale_v[b:b + 1], r, bits, block)
                    for i in range(4):
                        res[i][b] = one[i][0]
                    res[4][b] = pos + n
                    res[5][b] = False
            return tuple(res)
        out = list(orig(x, A_k, A_v, seq_lens, lat_k, scale_k, lat_v, scale_v, r, bits, block))
        if kind == "advance_by_one":
            out[4] = np.where(out[5], out[4], np.asarray(seq_lens, np.int32) + 1).astype(np.int32)
        return tuple(out)
    return f


@pytest.mark.parametrize("kind", ["batch_rows_swapped", "tokens_reversed", "accept_overflow", "advance_by_one"])
def test_prefill_mutants_are_caught(monkeypatch, kind):
    """A token written to another sequence's or another position's row, a
    block clipped at the capacity instead of refused, or the length advanced
    by one instead of T: at least one prefill pin must fail."""
    _patch(monkeypatch, "latent_prefill", _prefill_variant(kind))
    failed = 0
    for bits in (8, 4):
        try:
            P.test_prefill_equals_successive_appends(bits)
        except AssertionError:
            failed += 1
    for pin in (P.test_prefill_projection_is_one_dense_matmul, P.test_prefill_capacity_boundary_and_empty_block):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed > 0


def test_gqa_strided_grouping_mutant_is_caught(monkeypatch):
    """Query head g reading latent head g % Hkv (strided groups) instead of g // G."""
    def strided(q, lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r, bits, softmax_scale=None):
        B, Hq, Hd = q.shape
        Hkv = lat_k.shape[1]
        out = np.zeros((B, Hq, Hd))
        for b in range(B):
            for g in range(Hq):
                j = g % Hkv
                out[b, g], _ = OW.wsvd_decode_head(q[b, g], lat_k[b, j], scale_k[b, j], lat_v[b, j], scale_v[b, j],
                                                   Bk[j], Bv[j], int(seq_lens[b]), r, bits, softmax_scale)
        return out
    _patch(monkeypatch, "wsvd_decode_gqa", strided)
    with pytest.raises(AssertionError):
        P.test_gqa_matches_torch_grouped_sdpa(8)


def test_multi_token_visibility_mutant_is_caught(monkeypatch):
    """Every query of the block seeing the whole block (no causal step) must fail."""
    def no_causal(q, lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r, bits, softmax_scale=None):
        return np.stack([OW.wsvd_decode_gqa(q[:, t], lat_k, scale_k, lat_v, scale_v, Bk, Bv, seq_lens, r, bits,
                                            softmax_scale) for t in range(q.shape[1])], axis=1)
    _patch(monkeypatch, "wsvd_decode_multi", no_causal)
    with pytest.raises(AssertionError):
        P.test_multi_token_decode_is_causal_inside_the_block()
