"""The latent rotation S2 folded into the factors (wsvd_fold_latent_rotation):
the GPU's A . S2 and S2^T . B against the oracle's (fp16 results within one
unit in the last place of the correctly rounded value), and the step run on the
folded weights against the oracle run on the same folded weights."""
import numpy as np
import pytest
import torch

import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, dev, q_tensor
from oracle import wsvd_oracle as O

pytestmark = pytest.mark.gpu


def _ulp_diff(a16: np.ndarray, b16: np.ndarray) -> np.ndarray:
    """Distance in fp16 units in the last place (same-sign ordering)."""
    ai = a16.astype(np.float16).view(np.int16).astype(np.int32)
    bi = b16.astype(np.float16).view(np.int16).astype(np.int32)
    ai = np.where(ai < 0, -32768 - ai, ai)
    bi = np.where(bi < 0, -32768 - bi, bi)
    return np.abs(ai - bi)


@pytest.mark.parametrize("w", [WL.PR1, WL.LLAVA7B, WL.LONG[64].with_(E=512)])
def test_fold_matches_oracle(w):
    ai = WL.append_inputs(w, seed=2, steps=1)
    d = WL.decode_inputs(w.with_(L_cap=8, lens=8), seed=2)
    s2k, s2v = WL.latent_rotation(w, 2, "k"), WL.latent_rotation(w, 2, "v")
    out = W.wsvd_fold_latent_rotation(dev(s2k), dev(s2v), dev(ai.A_k), dev(ai.A_v), dev(d.Bk), dev(d.Bv))
    torch.cuda.synchronize()
    ak, bk = O.fold_latent_rotation(ai.A_k, d.Bk, s2k)
    av, bv = O.fold_latent_rotation(ai.A_v, d.Bv, s2v)
    for g, o in zip(out, (ak, av, bk, bv)):
        diff = _ulp_diff(g.cpu().numpy(), o)
        assert diff.max() <= 1, diff.max()


def test_step_on_folded_weights_matches_oracle():
    w = WL.LLAVA7B.with_(L_cap=1608)
    lens0 = [1599]
    d = WL.decode_inputs(w, seed=4, lens=np.asarray(lens0) + 1)
    d.lat_k[0, :, lens0[0]:] = 0
    d.lat_v[0, :, lens0[0]:] = 0
    d.scale_k[0, :, lens0[0]:] = 0
    d.scale_v[0, :, lens0[0]:] = 0
    d.seq_lens[:] = lens0
    ai = WL.append_inputs(w, seed=4, steps=1)
    s2k, s2v = WL.latent_rotation(w, 4, "k"), WL.latent_rotation(w, 4, "v")
    A_k, A_v, B_k, B_v = W.wsvd_fold_latent_rotation(dev(s2k), dev(s2v), dev(ai.A_k), dev(ai.A_v), dev(d.Bk),
                                                     dev(d.Bv))
    st = dict(lat_k=dev(d.lat_k), lat_v=dev(d.lat_v), sk=dev(d.scale_k), sv=dev(d.scale_v), lens=dev(d.seq_lens))
    out = W.wsvd_append_and_decode(q_tensor(ai.x_bits[0], "bf16"), A_k, A_v, st["lens"], st["lat_k"], st["lat_v"],
                                   st["sk"], st["sv"], q_tensor(d.q_bits, w.q_dtype), B_k, B_v, bits=w.bits)
    torch.cuda.synchronize()
    fA_k, fA_v, fB_k, fB_v = (t.cpu().numpy() for t in (A_k, A_v, B_k, B_v))
    olk, osk, olv, osv, olens, _, _, _ = O.latent_append(ai.x[0], fA_k, fA_v, d.seq_lens, d.lat_k, d.scale_k,
                                                         d.lat_v, d.scale_v, w.r, w.bits, w.hadamard_block)
    ref = O.wsvd_decode(d.q, olk, osk, olv, osv, fB_k, fB_v, olens, w.r, w.bits)
    assert_attention_close(out.cpu().numpy(), ref, "step on folded weights")
