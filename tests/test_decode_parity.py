"""GPU parity of wsvd_decode_attention against the float64 oracle.

Every case runs the CUDA path through the C ABI on seeded inputs and compares
element by element with the oracle (tolerance: max|gpu - oracle| <= 1e-3 *
max|oracle| + 1e-5 per (b, h) output); full-size long-context cases are
checked on sampled heads that the oracle recomputes one by one."""
import numpy as np
import pytest
import torch

import oracle as O
import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, decode_tensors, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from rank_kv_cache_wsvd_b200 import build
    build.build()
    W.load()


def run_gpu(d: WL.DecodeInputs, softmax_scale=0.0, reps=1):
    t = decode_tensors(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(reps):
        out = W.wsvd_decode_attention(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"],
                                      t["B_v"], t["seq_lens"], bits=d.w.bits, softmax_scale=softmax_scale, err=err)
        outs.append(out.cpu().numpy())
    torch.cuda.synchronize()
    return (outs[0] if reps == 1 else outs), int(err.item())


def oracle(d: WL.DecodeInputs, softmax_scale=None):
    return O.wsvd_decode(d.q, d.lat_k, d.scale_k, d.lat_v, d.scale_v, d.Bk, d.Bv, d.seq_lens, d.w.r, d.w.bits,
                         softmax_scale)


@pytest.mark.parametrize("name", ["pr1", "llava7b", "ragged"])
def test_workload_full(name):
    d = WL.decode_inputs(WL.PRESETS[name], seed=0)
    gpu, err = run_gpu(d)
    assert err == 0
    assert_attention_close(gpu, oracle(d), name)


@pytest.mark.parametrize("r", [16, 32, 64])
def test_long_context_sampled_heads(r):
    """Full-size long-context decode (B=4, H=32, L=32768) in the bench's launch
    configuration; the oracle recomputes a sample of heads from their seeds."""
    w = WL.LONG[r]
    d = WL.decode_inputs(w, seed=0)
    gpu, err = run_gpu(d)
    assert err == 0 and np.all(np.isfinite(gpu))
    for b, h in [(0, 0), (1, 17), (2, 31), (3, 8), (3, 30)]:
        lk, sk, lv, sv = WL.latent_cache_block(w, 0, b, h)
        ref, _ = O.wsvd_decode_head(d.q[b, h], lk, sk, lv, sv, d.Bk[h], d.Bv[h], int(d.seq_lens[b]), r, 8)
        assert_attention_close(gpu[b, h][None], ref[None], f"long r{r} b{b} h{h}")


def test_comparison_shape_l2048_full():
    """The WSVD arm of the comparison workload at its own shape (B 8, H 32,
    r 32 int8, fp16 query, L 2048): every (b, h) against the oracle."""
    d = WL.decode_inputs(WL.CMP[2048], seed=0)
    gpu, err = run_gpu(d)
    assert err == 0
    assert_attention_close(gpu, oracle(d), "cmp L2048")


def test_comparison_shape_l8192_sampled_heads():
    """The WSVD arm at L 8192 (B 8, H 32) in the bench's launch configuration;
    the oracle recomputes a sample of heads from their seeds."""
    w = WL.CMP[8192]
    d = WL.decode_inputs(w, seed=0)
    gpu, err = run_gpu(d)
    assert err == 0 and np.all(np.isfinite(gpu))
    for b, h in [(0, 0), (2, 13), (5, 31), (7, 7), (7, 30)]:
        lk, sk, lv, sv = WL.latent_cache_block(w, 0, b, h)
        ref, _ = O.wsvd_decode_head(d.q[b, h], lk, sk, lv, sv, d.Bk[h], d.Bv[h], int(d.seq_lens[b]), w.r, 8)
        assert_attention_close(gpu[b, h][None], ref[None], f"cmp L8192 b{b} h{h}")


TINY = [1, 2, 3, 7, 8, 33, 255, 256, 257]


@pytest.mark.parametrize("L", TINY)
@pytest.mark.parametrize("bits,r", [(8, 16), (8, 32), (8, 64), (8, 128), (4, 32), (4, 64)])
def test_tiny_and_ragged_lengths(L, bits, r):
    L_cap = (L + 7) // 8 * 8 + 8
    w = WL.Workload("tiny", B=3, H=3, Hd=64, r=r, bits=bits, L_cap=L_cap, lens=L, q_dtype="bf16")
    d = WL.decode_inputs(w, seed=L * 7 + r + bits, lens=[L, max(1, L // 2), min(L_cap, L + 3)])
    gpu, err = run_gpu(d)
    assert err == 0
    assert_attention_close(gpu, oracle(d), f"L={L} r={r} bits={bits}")


@pytest.mark.parametrize("Hd", [32, 64, 128, 256])
def test_head_dims_and_custom_scale(Hd):
    w = WL.Workload("hd", B=2, H=2, Hd=Hd, r=32, bits=8, L_cap=520, lens=(100, 520))
    d = WL.decode_inputs(w, seed=Hd)
    gpu, err = run_gpu(d, softmax_scale=0.05)
    assert err == 0
    assert_attention_close(gpu, oracle(d, softmax_scale=0.05), f"Hd={Hd}")


def test_poisoned_padding_is_bit_exact():
    """Rows past each sequence's length hold extreme codes and NaN/Inf scales;
    the outputs must be bitwise identical to the zero-padded cache."""
    for bits, r in [(8, 32), (4, 32), (8, 16)]:
        w = WL.Workload("poison", B=7, H=4, Hd=128, r=r, bits=bits, L_cap=1024, lens=(1, 1000))
        clean, e1 = run_gpu(WL.decode_inputs(w, seed=5))
        dirty, e2 = run_gpu(WL.decode_inputs(w, seed=5, poison=True))
        assert e1 == 0 and e2 == 0
        assert np.array_equal(clean.view(np.uint32), dirty.view(np.uint32)), (bits, r)


def test_deterministic():
    d = WL.decode_inputs(WL.RAGGED.with_(B=5), seed=3)
    (a, b), err = run_gpu(d, reps=2)
    assert err == 0 and np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_empty_and_out_of_range_lengths():
    w = WL.Workload("edge", B=4, H=2, Hd=64, r=32, bits=8, L_cap=64, lens=64)
    d = WL.decode_inputs(w, seed=1, lens=[0, 64, 5, 64])
    gpu, err = run_gpu(d)
    assert err == 0
    assert np.all(gpu[0] == 0)
    assert_attention_close(gpu[1:], oracle(d)[1:], "edge")
    # a length beyond L_cap is flagged on the device and gives zeros
    d.seq_lens[:] = [3, 65, -1, 64]
    gpu, err = run_gpu(d)
    assert err & 1
    assert np.all(gpu[1] == 0) and np.all(gpu[2] == 0)
    ref = oracle(WL.DecodeInputs(d.w, np.array([3, 0, 0, 64], np.int32), d.q, d.q_bits, d.lat_k, d.scale_k,
                                 d.lat_v, d.scale_v, d.Bk, d.Bv))
    assert_attention_close(gpu[[0, 3]], ref[[0, 3]], "edge-valid")


def test_output_and_workspace_guards():
    """Writes stay inside out[B][H][Hd] and inside the documented workspace size."""
    d = WL.decode_inputs(WL.PR1, seed=2)
    t = decode_tensors(d)
    B, H, Hd = d.q.shape
    n_out = B * H * Hd
    big = torch.full((n_out + 4096,), float("nan"), dtype=torch.float32, device="cuda")
    out = big[:n_out].view(B, H, Hd)
    need = W.wsvd_decode_workspace_size(B, H, d.w.r)
    ws_big = torch.full((need + 4096,), 0xA5, dtype=torch.uint8, device="cuda")
    W.wsvd_decode_attention(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                            t["seq_lens"], bits=8, out=out, workspace_buf=ws_big[:need])
    torch.cuda.synchronize()
    assert torch.isnan(big[n_out:]).all()
    assert (ws_big[need:] == 0xA5).all()
    assert_attention_close(out.cpu().numpy(), oracle(d), "guards")


def test_identity_factor_matches_gpu_dense_path():
    """r = Hd with B = I and power-of-two scales: the latents are exactly fp16 K
    and V, so the low-rank path must agree with the dense path on the GPU."""
    rng = np.random.default_rng(9)
    B, H, Hd, L = 2, 4, 64, 304
    Q = 127
    ck = rng.integers(-Q, Q + 1, size=(B, H, L, Hd))
    cv = rng.integers(-Q, Q + 1, size=(B, H, L, Hd))
    sk = (2.0 ** rng.integers(-9, -5, size=(B, H, L))).astype(np.float16)
    sv = (2.0 ** rng.integers(-9, -5, size=(B, H, L))).astype(np.float16)
    q = rng.standard_normal((B, H, Hd)).astype(np.float16)
    lens = np.array([300, 123], np.int32)
    I = np.broadcast_to(np.eye(Hd, dtype=np.float16), (H, Hd, Hd)).copy()
    lat_k, lat_v = O.pack_codes(ck, 8), O.pack_codes(cv, 8)
    out = W.wsvd_decode_attention(dev(q), dev(lat_k), dev(lat_v), dev(sk), dev(sv), dev(I), dev(I), dev(lens), 8)
    K = (ck * sk[..., None].astype(np.float64)).astype(np.float16)
    V = (cv * sv[..., None].astype(np.float64)).astype(np.float16)
    dense = W.dense_decode_attention(dev(q), dev(K), dev(V), dev(lens))
    torch.cuda.synchronize()
    ref = O.wsvd_decode(q, lat_k, sk, lat_v, sv, I, I, lens, Hd, 8)
    assert_attention_close(out.cpu().numpy(), ref, "identity")
    assert_attention_close(dense.cpu().numpy(), ref, "identity-dense")
    assert_attention_close(out.cpu().numpy(), dense.cpu().numpy(), "wsvd-vs-dense")
