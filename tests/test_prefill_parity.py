"""GPU parity of wsvd_latent_prefill (a block of T tokens per sequence) against
the float64 oracle: codes exact except counted +-1 rounding ties, scales exact
except counted fp16 rounding ties, only rows seq_lens[b] .. seq_lens[b] + T - 1
written (every other byte of a poisoned cache unchanged), seq_lens advanced by
T, refused blocks flagged and untouched."""
import numpy as np
import pytest
import torch

import oracle as O
import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import compare_codes, dev, q_tensor, unpack

pytestmark = pytest.mark.gpu

# Tie windows of the prefill, the same as the fp32 paths': a scale may differ
# by one fp16 step only where the oracle's fp32 ratio max|c| / Q lies within
# 2^-20 (relative) of an fp16 rounding midpoint, a code by one only where its
# ratio is within 1e-3 of a half step.  (Each 64-wide k-tile of the hi half
# is summed from zero on the tensor cores and the k-tiles are added with
# round-to-nearest, which keeps the error in c near 1e-7 of max|c|.)
SCALE_TOL = 2.0 ** -20
CODE_TOL = 1e-3


def tie_bounds(n_rows: int, r: int):
    """Upper bounds on the counted ties of n_rows quantised rows of r codes.
    Scales: fp16 midpoints lie 2^-11 .. 2^-10 apart relative to the value, so
    at most a fraction 2 * SCALE_TOL * 2^11 = 2^-8 of the ratios falls inside
    the window; that many rows may flip.  Codes: a window of 2 * CODE_TOL of
    every unit step holds at most that fraction of the n_rows * r codes."""
    return max(4, int(n_rows * r * 2 * CODE_TOL)), max(4, int(n_rows * 2 * SCALE_TOL * 2 ** 11))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from rank_kv_cache_wsvd_b200 import build
    build.build()
    W.load()


def _run(w: WL.Workload, T: int, lens0, bits=None, blk=None, x_dtype="bf16", seed=0):
    bits = w.bits if bits is None else bits
    blk = w.hadamard_block if blk is None else blk
    pi = WL.prefill_inputs(w, seed=seed, T=T)
    rng = np.random.default_rng(seed + 7)
    rb = w.r * bits // 8
    lat_k = rng.integers(0, 256, size=(w.B, w.H, w.L_cap, rb), dtype=np.uint8)
    lat_v = rng.integers(0, 256, size=(w.B, w.H, w.L_cap, rb), dtype=np.uint8)
    sc_k = rng.uniform(0, 1, (w.B, w.H, w.L_cap)).astype(np.float16)
    sc_v = rng.uniform(0, 1, (w.B, w.H, w.L_cap)).astype(np.float16)
    lens = np.asarray(lens0, np.int32)
    x_vals = pi.x
    if x_dtype == "bf16":
        x = q_tensor(pi.x_bits, "bf16")
    else:  # the same values rounded to fp16 (both sides see the fp16 values)
        x16 = pi.x.astype(np.float16)
        x_vals = x16.astype(np.float32)
        x = q_tensor(x16.view(np.uint16), "fp16")
    g = dict(lat_k=dev(lat_k), lat_v=dev(lat_v), sk=dev(sc_k), sv=dev(sc_v), lens=dev(lens))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    W.wsvd_latent_prefill(x, dev(pi.A_k), dev(pi.A_v), g["lens"], g["lat_k"], g["lat_v"], g["sk"], g["sv"],
                          bits=bits, hadamard_block=blk, err=err)
    torch.cuda.synchronize()
    olk, osk, olv, osv, olens, oerr, ck, cv = O.latent_prefill(x_vals, pi.A_k, pi.A_v, lens, lat_k, sc_k, lat_v,
                                                               sc_v, w.r, bits, blk)
    gl = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.array_equal(gl["lens"], olens), (gl["lens"], olens)
    ties = [0, 0]
    stats = {}
    written = np.zeros((w.B, w.L_cap), bool)
    for b in range(w.B):
        pos = int(lens[b])
        if oerr[b]:
            continue
        written[b, pos:pos + T] = True
        for which, c in (("k", ck), ("v", cv)):
            gc = unpack(gl["lat_" + which][b, :, pos:pos + T], w.r, bits)         # [H][T][r]
            oc = unpack((olk if which == "k" else olv)[b, :, pos:pos + T], w.r, bits)
            os_ = (osk if which == "k" else osv)[b, :, pos:pos + T]
            t = compare_codes(gc, gl["s" + which][b, :, pos:pos + T], oc, os_, c[b].transpose(1, 0, 2), bits,
                              tie_tol=CODE_TOL, scale_tol=SCALE_TOL, stats=stats)
            ties[0] += t[0]
            ties[1] += t[1]
    # every byte outside the written rows is what it was before the call
    for key, ref in (("lat_k", lat_k), ("lat_v", lat_v), ("sk", sc_k), ("sv", sc_v)):
        a = gl[key].view(np.uint8) if key.startswith("lat") else gl[key].view(np.uint16)
        r_ = ref.view(np.uint8) if key.startswith("lat") else ref.view(np.uint16)
        keep = ~written[:, None, :]
        assert np.array_equal(np.where(keep[..., None] if a.ndim == 4 else keep, a, 0),
                              np.where(keep[..., None] if r_.ndim == 4 else keep, r_, 0)), key
    print(f"prefill {w.name} T={T}: code ties {ties[0]}, scale ties {ties[1]}, largest distance to a tie "
          f"(scale, relative) {stats.get('scale_dist', 0.0):.3g}, (code, steps) {stats.get('code_dist', 0.0):.3g}")
    return ties, int(err.item()), gl, bool(oerr.any())


def test_llava_image_block_576_tokens():
    """The 576 image tokens of the LLaVA-7B-shaped layer in one call (B 1, H 32,
    E 4096, r 32, int8, 128-block Hadamard): five 128-row tiles (the last one
    ragged) x 16 column tiles of 128."""
    w = WL.LLAVA7B
    ties, err, g, _ = _run(w, 576, [0], seed=3)
    assert err == 0 and list(g["lens"]) == [576]
    code_bound, scale_bound = tie_bounds(576 * w.H * 2, w.r)
    assert ties[0] <= code_bound and ties[1] <= scale_bound, (ties, code_bound, scale_bound)


def test_ragged_rows_int4_and_exact_fit():
    """B 3, T 37 (111 token rows: a partial second row tile), int4 r 16, one
    sequence filling its cache exactly (27 + 37 = 64 = L_cap)."""
    w = WL.Workload("pf-ragged", B=3, H=4, Hd=64, r=16, bits=4, L_cap=64, lens=0, E=512)
    ties, err, g, _ = _run(w, 37, [0, 20, 27], seed=5)
    assert err == 0 and list(g["lens"]) == [37, 57, 64]


@pytest.mark.parametrize("H,r,bits", [(5, 64, 8), (5, 16, 8), (2, 128, 8), (3, 8, 4), (6, 32, 4)])
def test_column_tiles_heads_and_formats(H, r, bits):
    """Column tiles that straddle the K / V boundary (H 5, r 64: columns 256..383
    hold the last K head and the first V head), a partial last column tile
    (H 5, r 16: 160 columns), one head per tile (r 128), r 8 int4 rows of 4 bytes."""
    w = WL.Workload("pf-cols", B=2, H=H, Hd=64, r=r, bits=bits, L_cap=16, lens=0, E=256)
    ties, err, g, _ = _run(w, 5, [0, 9], seed=H * 100 + r)
    assert err == 0 and list(g["lens"]) == [5, 14]


def test_wide_tiles_of_eight_small_heads():
    """r 16 int4 with 128-column tiles (eight heads per tile): 4096 token rows
    over 16 heads fill the device with the wide tiles."""
    w = WL.Workload("pf-wide", B=2, H=16, Hd=64, r=16, bits=4, L_cap=2100, lens=0, E=256)
    ties, err, g, _ = _run(w, 2048, [0, 52], seed=21)
    assert err == 0 and list(g["lens"]) == [2048, 2100]
    code_bound, scale_bound = tie_bounds(2048 * w.B * w.H * 2, w.r)
    assert ties[0] <= code_bound and ties[1] <= scale_bound, (ties, code_bound, scale_bound)


def test_odd_k_tile_count_repeats_bit_for_bit():
    """E 1152 (18 k-tiles of 64, not a power of two) over 300 token rows (a
    ragged third row tile) and 8 heads; a second call on the same inputs
    writes the same bytes."""
    w = WL.Workload("pf-oddk", B=3, H=8, Hd=64, r=32, bits=8, L_cap=128, lens=0, E=1152)
    ties, err, g, _ = _run(w, 100, [0, 5, 28], seed=31)
    assert err == 0 and list(g["lens"]) == [100, 105, 128]
    ties2, err2, g2, _ = _run(w, 100, [0, 5, 28], seed=31)
    assert err2 == 0
    for k in ("lat_k", "lat_v", "sk", "sv"):
        assert np.array_equal(g[k].view(np.uint8), g2[k].view(np.uint8)), k


@pytest.mark.parametrize("E,blk,x_dtype", [(256, 1, "fp16"), (1024, 256, "bf16"), (2048, 64, "bf16"),
                                           (512, 1024 // 2, "fp16")])
def test_rotation_blocks_and_input_dtypes(E, blk, x_dtype):
    w = WL.Workload("pf-rot", B=2, H=3, Hd=64, r=32, bits=8, L_cap=12, lens=0, E=E)
    ties, err, g, _ = _run(w, 6, [0, 3], blk=blk, x_dtype=x_dtype, seed=E + blk)
    assert err == 0 and list(g["lens"]) == [6, 9]


def test_outlier_channels_long_context_recipe():
    """The long-context recipe's activations (0.1% of E channels x50) through
    the per-token power-of-two split: r 64, B 4, 64 tokens each."""
    w = WL.LONG[64].with_(L_cap=160)
    ties, err, g, _ = _run(w, 64, [0, 10, 96, 50], seed=11)
    assert err == 0 and list(g["lens"]) == [64, 74, 160, 114]
    code_bound, scale_bound = tie_bounds(64 * w.B * w.H * 2, w.r)
    assert ties[0] <= code_bound and ties[1] <= scale_bound, (ties, code_bound, scale_bound)


def test_refused_blocks_are_flagged_and_untouched():
    w = WL.Workload("pf-full", B=3, H=2, Hd=64, r=32, bits=8, L_cap=16, lens=0, E=256)
    ties, err, g, refused = _run(w, 8, [9, 8, -1], seed=2)  # 9 + 8 > 16 refused; 8 + 8 = 16 fits; -1 refused
    assert refused and err & 2
    assert list(g["lens"]) == [9, 16, -1]


def test_zero_tokens_is_a_no_op_and_zero_rows_give_zero_scale():
    w = WL.Workload("pf-zero", B=1, H=2, Hd=64, r=32, bits=8, L_cap=8, lens=0, E=256)
    lat = torch.full((1, 2, 8, 32), 0x55, dtype=torch.uint8, device="cuda")
    lat_v = lat.clone()
    sk = torch.ones((1, 2, 8), dtype=torch.float16, device="cuda")
    sv = sk.clone()
    lens = torch.tensor([2], dtype=torch.int32, device="cuda")
    A = torch.randn((2, 256, 32), device="cuda").half()
    W.wsvd_latent_prefill(torch.zeros((1, 0, 256), dtype=torch.bfloat16, device="cuda"), A, A, lens, lat, lat_v,
                          sk, sv, bits=8)
    torch.cuda.synchronize()
    assert int(lens.item()) == 2 and bool((lat == 0x55).all()) and bool((sk == 1).all())
    W.wsvd_latent_prefill(torch.zeros((1, 3, 256), dtype=torch.bfloat16, device="cuda"), A, A, lens, lat, lat_v,
                          sk, sv, bits=8)
    torch.cuda.synchronize()
    assert int(lens.item()) == 5
    assert bool((lat[0, :, 2:5] == 0).all()) and bool((sk[0, :, 2:5] == 0).all())
    assert bool((lat[0, :, :2] == 0x55).all()) and bool((lat[0, :, 5:] == 0x55).all())


def test_prefill_then_decode_matches_oracle():
    """The cache the prefill writes is the one the decode reads: prefill a
    576-token image block, append nothing, attend with the LLaVA query."""
    w = WL.LLAVA7B.with_(L_cap=640)
    pi = WL.prefill_inputs(w, seed=4, T=576)
    rb = w.r
    zeros = lambda: torch.zeros((1, w.H, w.L_cap, rb), dtype=torch.uint8, device="cuda")
    lk, lv = zeros(), zeros()
    sk = torch.zeros((1, w.H, w.L_cap), dtype=torch.float16, device="cuda")
    sv = sk.clone()
    lens = torch.zeros(1, dtype=torch.int32, device="cuda")
    W.wsvd_latent_prefill(q_tensor(pi.x_bits, "bf16"), dev(pi.A_k), dev(pi.A_v), lens, lk, lv, sk, sv, bits=8)
    d = WL.decode_inputs(w, seed=4, lens=np.array([576]))
    out = W.wsvd_decode_attention(q_tensor(d.q_bits, w.q_dtype), lk, lv, sk, sv, dev(d.Bk), dev(d.Bv), lens, bits=8)
    torch.cuda.synchronize()
    from gpu_util import assert_attention_close
    ref = O.wsvd_decode(d.q, lk.cpu().numpy(), sk.cpu().numpy(), lv.cpu().numpy(), sv.cpu().numpy(), d.Bk, d.Bv,
                        lens.cpu().numpy(), w.r, 8)
    assert_attention_close(out.cpu().numpy(), ref, "prefill -> decode")
