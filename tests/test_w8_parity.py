"""Int8 weights (W8): the decode, the latent append and the one-call step with
A_k, A_v, B_k, B_v stored as int8 plus one fp32 scale per output column,
checked against the oracle run on the dequantised weights (attention within
the tolerance, codes exact except counted rounding ties), and the one-call step
against the two W8 calls bit for bit."""
import numpy as np
import pytest
import torch

import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, compare_codes, decode_tensors, dev, q_tensor, unpack
from oracle import wsvd_oracle as O

pytestmark = pytest.mark.gpu


def _w8(Wf):
    q, s = WL.quantize_weights_w8(Wf)
    return q, s, O.dequantize_weights(q, s)


@pytest.mark.parametrize("name,w", [
    ("llava7b", WL.LLAVA7B),                                  # cluster path, int8, bf16 q
    ("pr1-hd64", WL.PR1),                                     # cluster path, Hd 64, r 16
    ("ragged-int4", WL.RAGGED.with_(B=6)),                    # split-L grid, int4, fp16 q
    ("long-r64", WL.LONG[64].with_(B=2, L_cap=4096, lens=4096)),  # split-L grid, two lanes per token
])
def test_w8_decode_matches_oracle(name, w):
    d = WL.decode_inputs(w, seed=5)
    t = decode_tensors(d)
    bkq, sbk, bk = _w8(d.Bk)
    bvq, sbv, bv = _w8(d.Bv)
    out = W.wsvd_decode_attention_w8(t["q"], t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], dev(bkq), dev(bvq),
                                     dev(sbk), dev(sbv), t["seq_lens"], bits=w.bits)
    torch.cuda.synchronize()
    ref = O.wsvd_decode(d.q, d.lat_k, d.scale_k, d.lat_v, d.scale_v, bk, bv, d.seq_lens, w.r, w.bits)
    assert_attention_close(out.cpu().numpy(), ref, f"w8 decode {name}")


def _empty_cache(w, bits):
    rb = w.r * bits // 8
    return (np.zeros((w.B, w.H, w.L_cap, rb), np.uint8), np.zeros((w.B, w.H, w.L_cap), np.float16),
            np.zeros((w.B, w.H, w.L_cap, rb), np.uint8), np.zeros((w.B, w.H, w.L_cap), np.float16))


@pytest.mark.parametrize("name,w,lens0", [
    ("llava7b", WL.LLAVA7B.with_(L_cap=1608), [1599]),
    ("long-r32-b4", WL.LONG[32].with_(L_cap=64), [0, 5, 63, 17]),
    ("int4-r32-b3", WL.RAGGED.with_(B=3, E=1024, L_cap=64), [1, 2, 3]),
    ("r64-b16", WL.LONG[64].with_(B=16, E=512, L_cap=16), list(range(16))),
])
def test_w8_append_matches_oracle(name, w, lens0):
    ai = WL.append_inputs(w, seed=9, steps=1)
    akq, sak, ak = _w8(ai.A_k)
    avq, sav, av = _w8(ai.A_v)
    lk, sk, lv, sv = _empty_cache(w, w.bits)
    g = dict(lat_k=dev(lk), lat_v=dev(lv), sk=dev(sk), sv=dev(sv), lens=dev(np.asarray(lens0, np.int32)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    W.wsvd_latent_append_w8(q_tensor(ai.x_bits[0], "bf16"), dev(akq), dev(avq), dev(sak), dev(sav), g["lens"],
                            g["lat_k"], g["lat_v"], g["sk"], g["sv"], bits=w.bits, hadamard_block=w.hadamard_block,
                            err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    olk, osk, olv, osv, olens, _, ck, cv = O.latent_append(ai.x[0], ak, av, np.asarray(lens0, np.int32), lk, sk, lv,
                                                           sv, w.r, w.bits, w.hadamard_block)
    gl = {k: v.cpu().numpy() for k, v in g.items()}
    assert np.array_equal(gl["lens"], olens)
    for b, pos in enumerate(lens0):
        for which, glat, gs, olat, os_, c in (("k", gl["lat_k"], gl["sk"], olk, osk, ck),
                                               ("v", gl["lat_v"], gl["sv"], olv, osv, cv)):
            compare_codes(unpack(glat[b, :, pos], w.r, w.bits), gs[b, :, pos], unpack(olat[b, :, pos], w.r, w.bits),
                          os_[b, :, pos], c[b], w.bits)


def test_w8_step_equals_the_two_w8_calls_and_the_oracle():
    w = WL.LLAVA7B
    assert W.wsvd_step_launch_count(w.B, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap, w.hadamard_block, w8=True) == 1
    w4 = WL.RAGGED.with_(B=1, H=8, E=2048, L_cap=1024)
    assert W.wsvd_step_launch_count(w4.B, w4.H, w4.Hd, w4.E, w4.r, w4.bits, w4.L_cap, w4.hadamard_block, w8=True) == 1
    for w, lens0 in ((WL.LLAVA7B.with_(L_cap=1608), [1599]),                    # one kernel (cluster decode)
                     (WL.RAGGED.with_(B=1, H=8, E=2048, L_cap=1024), [700]),     # one kernel, int4 cache
                     (WL.LONG[32].with_(L_cap=8192), [8000, 8191, 100, 4095])):  # split-L grid
        d = WL.decode_inputs(w, seed=21, lens=np.asarray(lens0) + 1)
        for b, n in enumerate(lens0):
            d.lat_k[b, :, n:] = 0
            d.lat_v[b, :, n:] = 0
            d.scale_k[b, :, n:] = 0
            d.scale_v[b, :, n:] = 0
        d.seq_lens[:] = lens0
        ai = WL.append_inputs(w, seed=21, steps=1)
        akq, sak, ak = _w8(ai.A_k)
        avq, sav, av = _w8(ai.A_v)
        bkq, sbk, bk = _w8(d.Bk)
        bvq, sbv, bv = _w8(d.Bv)
        wts = [dev(v) for v in (akq, avq, sak, sav, bkq, bvq, sbk, sbv)]
        x = q_tensor(ai.x_bits[0], "bf16")
        q = q_tensor(d.q_bits, w.q_dtype)

        def state():
            return dict(lat_k=dev(d.lat_k), lat_v=dev(d.lat_v), sk=dev(d.scale_k), sv=dev(d.scale_v),
                        lens=dev(d.seq_lens))

        two, one = state(), state()
        W.wsvd_latent_append_w8(x, wts[0], wts[1], wts[2], wts[3], two["lens"], two["lat_k"], two["lat_v"], two["sk"],
                                two["sv"], bits=w.bits)
        out2 = W.wsvd_decode_attention_w8(q, two["lat_k"], two["lat_v"], two["sk"], two["sv"], wts[4], wts[5], wts[6],
                                          wts[7], two["lens"], bits=w.bits)
        out1 = W.wsvd_append_and_decode_w8(x, wts[0], wts[1], wts[2], wts[3], one["lens"], one["lat_k"], one["lat_v"],
                                           one["sk"], one["sv"], q, wts[4], wts[5], wts[6], wts[7], bits=w.bits)
        torch.cuda.synchronize()
        for k in ("lat_k", "lat_v", "sk", "sv", "lens"):
            assert torch.equal(one[k], two[k]), k
        assert torch.equal(out1, out2)
        olk, osk, olv, osv, olens, _, _, _ = O.latent_append(ai.x[0], ak, av, d.seq_lens, d.lat_k, d.scale_k, d.lat_v,
                                                             d.scale_v, w.r, w.bits, w.hadamard_block)
        ref = O.wsvd_decode(d.q, olk, osk, olv, osv, bk, bv, olens, w.r, w.bits)
        assert_attention_close(out1.cpu().numpy(), ref, "w8 step")


def test_w8_entry_points_reject_missing_scales():
    w = WL.PR1
    d = WL.decode_inputs(w, seed=1)
    t = decode_tensors(d)
    bkq, sbk, _ = _w8(d.Bk)
    lib = W.load()
    p = lambda v: v.data_ptr()
    st = lib.wsvd_decode_attention_w8(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap, p(t["seq_lens"]), p(t["q"]), 0,
                                      p(t["lat_k"]), p(t["lat_v"]), p(t["scale_k"]), p(t["scale_v"]),
                                      p(dev(bkq)), p(dev(bkq)), None, None, 0.0, p(torch.empty(w.B, w.H, w.Hd,
                                                                                               device="cuda")),
                                      p(W.workspace(W.wsvd_decode_workspace_size(w.B, w.H, w.r))),
                                      W.wsvd_decode_workspace_size(w.B, w.H, w.r), None, None)
    assert st == 1  # WSVD_ERR_INVALID_ARG
