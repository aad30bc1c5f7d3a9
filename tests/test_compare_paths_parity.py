"""GPU parity of the two in-library comparison paths against the oracle:
the dense fp16 flash-decode and the conventional shared-latent SVD decode."""
import numpy as np
import pytest
import torch

import oracle as O
import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, dev, q_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from rank_kv_cache_wsvd_b200 import build
    build.build()
    W.load()


def run_dense(w, lens=None, seed=0):
    d = WL.dense_inputs(w, seed=seed, lens=lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = W.dense_decode_attention(q_tensor(d["q_bits"], w.q_dtype), dev(d["K"]), dev(d["V"]), dev(d["seq_lens"]),
                                   err=err)
    torch.cuda.synchronize()
    return d, out.cpu().numpy(), int(err.item())


def run_shared(w, lens=None, seed=0):
    d = WL.shared_inputs(w, seed=seed, lens=lens)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = W.shared_latent_svd_decode(q_tensor(d["q_bits"], w.q_dtype), dev(d["lat_k"]), dev(d["lat_v"]),
                                     dev(d["Bk"]), dev(d["Bv"]), dev(d["seq_lens"]), err=err)
    torch.cuda.synchronize()
    return d, out.cpu().numpy(), int(err.item())


def test_dense_full_l2048():
    w = WL.CMP[2048]
    d, gpu, err = run_dense(w)
    assert err == 0
    assert_attention_close(gpu, O.dense_decode(d["q"], d["K"], d["V"], d["seq_lens"]), "dense L2048")


def test_dense_l8192_sampled():
    w = WL.CMP[8192]
    d, gpu, err = run_dense(w)
    assert err == 0
    for b, h in [(0, 0), (3, 11), (7, 31)]:
        ref = O.dense_decode(d["q"][b:b + 1, h:h + 1], d["K"][b:b + 1, h:h + 1], d["V"][b:b + 1, h:h + 1],
                             d["seq_lens"][b:b + 1])
        assert_attention_close(gpu[b, h][None], ref[0], f"dense b{b} h{h}")


@pytest.mark.parametrize("Hd", [64, 128, 256])
def test_dense_ragged(Hd):
    w = WL.Workload("dense-ragged", B=5, H=3, Hd=Hd, r=32, bits=8, L_cap=520, lens=(1, 520))
    d, gpu, err = run_dense(w, seed=Hd)
    assert err == 0
    assert_attention_close(gpu, O.dense_decode(d["q"], d["K"], d["V"], d["seq_lens"]), f"dense Hd{Hd}")


@pytest.mark.parametrize("R", [128, 256, 512, 1024])
def test_shared_small_full(R):
    w = WL.Workload("shared-small", B=3, H=4, Hd=128, r=32, bits=8, L_cap=304, lens=(1, 300), R=R)
    d, gpu, err = run_shared(w, seed=R)
    assert err == 0
    ref = O.shared_latent_decode(d["q"], d["lat_k"], d["lat_v"], d["Bk"], d["Bv"], d["seq_lens"])
    assert_attention_close(gpu, ref, f"shared R{R}")


@pytest.mark.parametrize("L", [2048, 8192])
def test_shared_full_size_sampled(L):
    w = WL.CMP[L]
    d, gpu, err = run_shared(w)
    assert err == 0
    for b, h in [(0, 0), (5, 20), (7, 31)]:
        ref = O.shared_latent_decode(d["q"][b:b + 1, h:h + 1], d["lat_k"][b:b + 1], d["lat_v"][b:b + 1],
                                     d["Bk"][h:h + 1], d["Bv"][h:h + 1], d["seq_lens"][b:b + 1])
        assert_attention_close(gpu[b, h][None], ref[0], f"shared L{L} b{b} h{h}")
