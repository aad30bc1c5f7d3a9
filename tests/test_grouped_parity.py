"""GPU parity of the grouped-query / multi-token decode (wsvd_decode_gqa,
wsvd_decode_multi) against the float64 oracle's wsvd_decode_gqa and
wsvd_decode_multi: per output vector max|gpu - oracle| <= 1e-3 max|oracle| +
1e-5.  Query head g reads latent head g // G; query token t of a block of Tq
sees rows [0, len - Tq + 1 + t)."""
import numpy as np
import pytest
import torch

import oracle as O
import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, decode_tensors, dev, q_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from rank_kv_cache_wsvd_b200 import build
    build.build()
    W.load()


def _inputs(w: WL.Workload, Hq: int, Tq: int, seed: int, lens=None, poison=False):
    """Cache over w.H = Hkv latent heads; queries [B][Tq][Hq][Hd]."""
    d = WL.decode_inputs(w, seed=seed, lens=lens, poison=poison)
    q, qb = WL.multi_query(w, seed, Tq, Hq)
    return d, q, qb


def _run(d, qb, Tq, Hq, reps=1, softmax_scale=0.0):
    w = d.w
    t = decode_tensors(d)
    qt = q_tensor(qb, w.q_dtype)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(reps):
        if Tq == 1:
            out = W.wsvd_decode_gqa(qt[:, 0].contiguous(), t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"],
                                    t["B_k"], t["B_v"], t["seq_lens"], bits=w.bits, softmax_scale=softmax_scale,
                                    err=err)[:, None]
        else:
            out = W.wsvd_decode_multi(qt, t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                                      t["seq_lens"], bits=w.bits, softmax_scale=softmax_scale, err=err)
        outs.append(out.cpu().numpy())
    torch.cuda.synchronize()
    return (outs[0] if reps == 1 else outs), int(err.item())


def _oracle(d, q, softmax_scale=None):
    return O.wsvd_decode_multi(q, d.lat_k, d.scale_k, d.lat_v, d.scale_v, d.Bk, d.Bv, d.seq_lens, d.w.r, d.w.bits,
                               softmax_scale)


def _check(gpu, ref, what):
    B, Tq, Hq, Hd = ref.shape
    assert_attention_close(gpu.reshape(-1, Hd), ref.reshape(-1, Hd), what)


@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("Tq", [1, 4])
@pytest.mark.parametrize("bits", [8, 4])
def test_llava_shape(G, Tq, bits):
    """The LLaVA-7B-shaped layer (B 1, 32 query heads, Hd 128, r 32, 1600 cached
    tokens) with G query heads per latent head and Tq tokens per step."""
    Hq = 32
    w = WL.LLAVA7B.with_(H=Hq // G, bits=bits)
    d, q, qb = _inputs(w, Hq, Tq, seed=G * 10 + Tq + bits)
    gpu, err = _run(d, qb, Tq, Hq)
    assert err == 0
    _check(gpu, _oracle(d, q), f"llava G{G} Tq{Tq} int{bits}")


@pytest.mark.parametrize("bits,r", [(8, 16), (8, 32), (8, 64), (4, 32), (4, 64), (4, 128)])
@pytest.mark.parametrize("G,Tq", [(2, 3), (8, 4), (3, 1), (1, 7)])
def test_ragged_lengths_ranks_and_query_counts(bits, r, G, Tq):
    """Ragged lengths over several splits and a ragged last tile, every rank the
    kernel is built for, query counts that pad a chunk (6, 3, 7) or need two
    chunks of 16 (32)."""
    Hkv = 2
    Hq = G * Hkv
    w = WL.Workload("gq", B=4, H=Hkv, Hd=64, r=r, bits=bits, L_cap=1304, lens=1304, q_dtype="bf16")
    lens = [1304, 1, 130, 777]
    d, q, qb = _inputs(w, Hq, Tq, seed=r + bits + 7 * G + Tq, lens=lens)
    gpu, err = _run(d, qb, Tq, Hq)
    assert err == 0
    _check(gpu, _oracle(d, q), f"r{r} int{bits} G{G} Tq{Tq}")


def test_long_context_sampled():
    """B 2, L 32768, 4 latent heads of 8 query heads each, Tq 2: a many-split
    plan; the oracle checks a sample of (b, query token, head)."""
    w = WL.LONG[32].with_(B=2, H=4)
    Hq, Tq = 32, 2
    d, q, qb = _inputs(w, Hq, Tq, seed=5)
    gpu, err = _run(d, qb, Tq, Hq)
    assert err == 0 and np.all(np.isfinite(gpu))
    for b, t, hq in [(0, 0, 0), (0, 1, 13), (1, 0, 31), (1, 1, 8)]:
        hkv = hq // (Hq // w.H)
        n = int(d.seq_lens[b]) - Tq + 1 + t
        ref, _ = O.wsvd_decode_head(q[b, t, hq], d.lat_k[b, hkv], d.scale_k[b, hkv], d.lat_v[b, hkv],
                                    d.scale_v[b, hkv], d.Bk[hkv], d.Bv[hkv], n, w.r, w.bits)
        assert_attention_close(gpu[b, t, hq][None], ref[None], f"long b{b} t{t} h{hq}")


def test_queries_that_see_nothing_and_empty_sequences():
    """len < Tq leaves the first queries with no visible row (out = 0); len 0
    gives zeros; a length beyond L_cap is flagged and gives zeros."""
    w = WL.Workload("gq-edge", B=4, H=2, Hd=64, r=32, bits=8, L_cap=64, lens=64)
    Hq, Tq = 4, 4
    d, q, qb = _inputs(w, Hq, Tq, seed=3, lens=[2, 0, 64, 5])
    gpu, err = _run(d, qb, Tq, Hq)
    assert err == 0
    ref = _oracle(d, q)
    assert np.all(gpu[0, :2] == 0) and np.all(gpu[1] == 0)
    _check(gpu, ref, "edge")
    d.seq_lens[:] = [3, 65, -1, 64]
    gpu, err = _run(d, qb, Tq, Hq)
    assert err & 1
    assert np.all(gpu[1] == 0) and np.all(gpu[2] == 0)


def test_poisoned_padding_is_bit_exact_and_deterministic():
    for bits, r in [(8, 32), (4, 64)]:
        w = WL.Workload("gq-poison", B=3, H=2, Hd=128, r=r, bits=bits, L_cap=1024, lens=(1, 1000))
        _, _, qb = _inputs(w, 8, 2, seed=9)
        clean, e1 = _run(WL.decode_inputs(w, seed=9), qb, 2, 8, reps=2)
        dirty, e2 = _run(WL.decode_inputs(w, seed=9, poison=True), qb, 2, 8)
        assert e1 == 0 and e2 == 0
        assert np.array_equal(clean[0].view(np.uint32), clean[1].view(np.uint32)), "not deterministic"
        assert np.array_equal(clean[0].view(np.uint32), dirty.view(np.uint32)), (bits, r)


def test_single_query_matches_the_one_query_kernel():
    """G = 1, Tq = 1 is the plain decode: the tensor-core kernel and
    wsvd_decode_attention agree within the attention tolerance."""
    w = WL.RAGGED.with_(B=3)
    d, q, qb = _inputs(w, w.H, 1, seed=4)
    gpu, err = _run(d, qb, 1, w.H)
    assert err == 0
    t = decode_tensors(d)
    one = W.wsvd_decode_attention(q_tensor(qb[:, 0].copy(), w.q_dtype), t["lat_k"], t["lat_v"], t["scale_k"],
                                  t["scale_v"], t["B_k"], t["B_v"], t["seq_lens"], bits=w.bits).cpu().numpy()
    assert_attention_close(gpu[:, 0].reshape(-1, w.Hd), one.reshape(-1, w.Hd), "vs one-query kernel")
    _check(gpu, _oracle(d, q), "ragged G1")


def test_custom_softmax_scale_and_head_dims():
    for Hd in (32, 256):
        w = WL.Workload("gq-hd", B=2, H=2, Hd=Hd, r=32, bits=8, L_cap=520, lens=(100, 520))
        d, q, qb = _inputs(w, 4, 2, seed=Hd)
        gpu, err = _run(d, qb, 2, 4, softmax_scale=0.05)
        assert err == 0
        _check(gpu, _oracle(d, q, softmax_scale=0.05), f"Hd {Hd}")


def test_workspace_guard_and_counters_left_zero():
    """Writes stay inside the documented workspace; a second call on the same
    workspace (its counters left zero) gives the same bits."""
    w = WL.Workload("gq-ws", B=2, H=2, Hd=64, r=32, bits=8, L_cap=4096, lens=4096)
    Hq, Tq = 8, 2
    d, q, qb = _inputs(w, Hq, Tq, seed=1)
    t = decode_tensors(d)
    need = W.wsvd_decode_multi_workspace_size(w.B, Tq, Hq, w.H, w.r, w.L_cap)
    ws = torch.full((need + 4096,), 0, dtype=torch.uint8, device="cuda")
    ws[need:] = 0xA5
    qt = q_tensor(qb, w.q_dtype)
    outs = [W.wsvd_decode_multi(qt, t["lat_k"], t["lat_v"], t["scale_k"], t["scale_v"], t["B_k"], t["B_v"],
                                t["seq_lens"], bits=8, workspace_buf=ws[:need]).cpu().numpy() for _ in range(2)]
    torch.cuda.synchronize()
    assert (ws[need:] == 0xA5).all()
    assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))
    _check(outs[0], _oracle(d, q), "ws")
