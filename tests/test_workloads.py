"""Host-side checks of the seeded synthetic inputs (no GPU)."""
import numpy as np

import workloads as W


def test_presets_have_the_stated_shapes():
    p = W.PRESETS
    assert (p["pr1"].B, p["pr1"].H, p["pr1"].Hd, p["pr1"].r, p["pr1"].L_cap) == (1, 4, 64, 16, 256)
    assert (p["llava7b"].H, p["llava7b"].Hd, p["llava7b"].E, p["llava7b"].r, p["llava7b"].L_cap) == \
        (32, 128, 4096, 32, 1600)
    assert p["ragged"].bits == 4 and p["ragged"].lens == (1024, 4096) and p["ragged"].B == 16
    assert [p[f"long_r{r}"].r for r in (16, 32, 64)] == [16, 32, 64]
    assert p["long_r32"].L_cap == 32768 and p["long_r32"].append_steps == 64
    assert p["cmp_l8192"].R == 512 and p["cmp_l2048"].B == 8


def test_determinism_and_block_independence():
    w = W.PR1.with_(H=2, L_cap=32, lens=32)
    a = W.decode_inputs(w, seed=3)
    b = W.decode_inputs(w, seed=3)
    assert np.array_equal(a.lat_k, b.lat_k) and np.array_equal(a.scale_v, b.scale_v)
    lk, sk, lv, sv = W.latent_cache_block(w, 3, 0, 1)
    assert np.array_equal(lk, a.lat_k[0, 1]) and np.array_equal(sv, a.scale_v[0, 1])
    c = W.decode_inputs(w, seed=4)
    assert not np.array_equal(a.lat_k, c.lat_k)


def test_dtype_exactness():
    x = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    v, bits = W.to_dtype_exact(x, "bf16")
    assert np.array_equal(W.round_to_bf16(v), v)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), v)
    assert np.all(np.abs(v - x) <= np.abs(x) * 2.0 ** -8)
    v16, b16 = W.to_dtype_exact(x, "fp16")
    assert np.array_equal(b16.view(np.float16).astype(np.float32), v16)


def test_ragged_lengths_and_padding():
    w = W.RAGGED.with_(B=6, H=2, L_cap=64, lens=(3, 64))
    d = W.decode_inputs(w, seed=1)
    assert d.seq_lens.min() >= 3 and d.seq_lens.max() <= 64
    for b in range(w.B):
        n = d.seq_lens[b]
        assert np.all(d.lat_k[b, :, n:] == 0) and np.all(d.scale_k[b, :, n:] == 0)
    p = W.decode_inputs(w, seed=1, poison=True)
    for b in range(w.B):
        n = d.seq_lens[b]
        assert np.array_equal(p.lat_k[b, :, :n], d.lat_k[b, :, :n])
        if n < w.L_cap:
            assert np.all(p.lat_k[b, :, n:] == 0x77)
            assert np.isnan(p.scale_k[b, 0, n].astype(np.float32))


def test_synthetic_storage_is_close_to_the_latent():
    g = np.random.default_rng(2)
    x = g.standard_normal((100, 32))
    for bits in (8, 4):
        lat, s = W.synth_latent_storage(x, bits)
        Q = W.qmax(bits)
        if bits == 8:
            codes = lat.view(np.int8).astype(np.float64)
        else:
            lo = (lat & 0xF).astype(np.int64)
            hi = (lat >> 4).astype(np.int64)
            codes = np.empty((100, 32))
            codes[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
            codes[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
        err = np.abs(codes * s.astype(np.float64)[:, None] - x)
        assert np.all(err <= s.astype(np.float64)[:, None] * 0.51 + 1e-3 * np.abs(x)), bits
        assert np.all(np.abs(codes) <= Q)


def test_append_inputs_outliers():
    w = W.LONG[32].with_(B=2, append_steps=3)
    a = W.append_inputs(w, seed=0)
    assert a.x.shape == (3, 2, 4096) and a.A_k.shape == (32, 4096, 32)
    big = np.abs(a.x).max(axis=(0, 1)) > 20
    assert 1 <= big.sum() <= 8


def test_w8_weight_recipe_hits_the_code_range_per_column():
    """Per output column: every code in [-127, 127], the largest magnitude 127,
    and the dequantised matrix within half a step of the fp16 one."""
    ai = W.append_inputs(W.PR1, seed=0, steps=1)
    q, s = W.quantize_weights_w8(ai.A_k)
    assert q.dtype == np.int8 and s.dtype == np.float32 and s.shape == (W.PR1.H, W.PR1.r)
    assert np.abs(q.astype(int)).max() <= 127
    assert np.all(np.abs(q.astype(int)).max(axis=1) == 127)
    back = q.astype(np.float64) * s.astype(np.float64)[:, None, :]
    # half a step, plus the float32 rounding of w / scale (up to 127 * 2^-24 code units)
    assert np.all(np.abs(back - ai.A_k.astype(np.float64)) <= (0.5 + 1e-4) * s.astype(np.float64)[:, None, :])


def test_prefill_inputs_are_the_append_steps_as_one_block():
    """Token t of the prefill block is the activation of append step t (same seed),
    laid out [B][T][E]; the factors are the append's."""
    w = W.LONG[16].with_(B=3)
    p = W.prefill_inputs(w, seed=4, T=5)
    a = W.append_inputs(w, seed=4, steps=5)
    assert p.x.shape == (3, 5, 4096) and p.x_bits.shape == (3, 5, 4096)
    assert np.array_equal(p.x, a.x.transpose(1, 0, 2)) and np.array_equal(p.x_bits, a.x_bits.transpose(1, 0, 2))
    assert np.array_equal(p.A_k, a.A_k) and np.array_equal(p.A_v, a.A_v)
    assert p.x.flags["C_CONTIGUOUS"] and W.LLAVA7B.prefill_tokens == 576
