"""The one-call decode step, wsvd_append_and_decode: one kernel that appends
and attends (one sequence on the cluster decode path), or the latent append
followed by the decode launched behind it as a programmatic dependent.  Its
results must be those of the two calls made one after the other, bit for bit
(cache rows, scales, lengths, output), and the oracle's two steps within the
attention tolerance."""
import numpy as np
import pytest
import torch

import rank_kv_cache_wsvd_b200 as W
import workloads as WL
from gpu_util import assert_attention_close, dev, q_tensor
from oracle import wsvd_oracle as O

pytestmark = pytest.mark.gpu

CASES = {
    # one kernel (cluster decode path, B = 1): the new row in the last rank's chunk
    "llava7b": (WL.LLAVA7B.with_(L_cap=1608), [1599]),
    # one kernel: the new row is the first of rank 7's chunk (no cached rows before it there)
    "llava7b-chunk-start": (WL.LLAVA7B, [1400]),
    # one kernel: rank 4 owns the new row, ranks 5-7 hold no rows
    "llava7b-middle": (WL.LLAVA7B, [803]),
    # one kernel: the new row is the last of rank 6's chunk (the last lane of the tile)
    "llava7b-chunk-end": (WL.LLAVA7B, [1399]),
    # one kernel: empty cache, rank 0 (which also merges) owns the only row
    "llava7b-first-row": (WL.LLAVA7B, [0]),
    # one kernel, int4 cache, fp16 query
    "int4-one-kernel": (WL.RAGGED.with_(B=1, H=8, E=2048, L_cap=1024), [700]),
    # one kernel, two-CTA clusters (E 512 with 256-wide Hadamard blocks), x rotated in shared memory
    "two-rank": (WL.PR1.with_(r=32, E=512, hadamard_block=256, L_cap=256), [77]),
    # one kernel, one CTA per head
    "one-rank": (WL.PR1.with_(r=32, E=256, hadamard_block=256, L_cap=128), [100]),
    # persistent decode path, a length at the last free row and a short one
    "long-r32": (WL.LONG[32].with_(L_cap=8192), [8000, 8191, 100, 4095]),
    # int4 cache, fp16 query, ragged lengths
    "ragged-int4": (WL.RAGGED.with_(B=6, E=2048), [1023, 4095, 2000, 1, 3333, 64]),
    "pr1": (WL.PR1.with_(L_cap=264), [255]),
}


def _inputs(w, lens0, seed):
    d = WL.decode_inputs(w, seed=seed, lens=np.asarray(lens0) + 1)
    for b, n in enumerate(lens0):  # the row the append writes starts out empty
        d.lat_k[b, :, n:] = 0
        d.lat_v[b, :, n:] = 0
        d.scale_k[b, :, n:] = 0
        d.scale_v[b, :, n:] = 0
    d.seq_lens[:] = lens0
    ai = WL.append_inputs(w, seed=seed, steps=1)
    return d, ai


def _device_state(d):
    return dict(lat_k=dev(d.lat_k), lat_v=dev(d.lat_v), sk=dev(d.scale_k), sv=dev(d.scale_v), lens=dev(d.seq_lens))


@pytest.mark.parametrize("name", list(CASES))
def test_step_equals_append_then_decode(name):
    w, lens0 = CASES[name]
    d, ai = _inputs(w, lens0, seed=21)
    x = q_tensor(ai.x_bits[0], "bf16")
    A_k, A_v, B_k, B_v = dev(ai.A_k), dev(ai.A_v), dev(d.Bk), dev(d.Bv)
    q = q_tensor(d.q_bits, w.q_dtype)
    two, one = _device_state(d), _device_state(d)
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    err1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    W.wsvd_latent_append(x, A_k, A_v, two["lens"], two["lat_k"], two["lat_v"], two["sk"], two["sv"], bits=w.bits,
                         hadamard_block=w.hadamard_block, err=err2)
    out2 = W.wsvd_decode_attention(q, two["lat_k"], two["lat_v"], two["sk"], two["sv"], B_k, B_v, two["lens"],
                                   bits=w.bits, err=err2)
    for rep in range(2):  # the second call proves the workspaces were left zero
        st = _device_state(d) if rep else one
        out1 = W.wsvd_append_and_decode(x, A_k, A_v, st["lens"], st["lat_k"], st["lat_v"], st["sk"], st["sv"], q,
                                        B_k, B_v, bits=w.bits, hadamard_block=w.hadamard_block, err=err1)
        torch.cuda.synchronize()
        assert int(err1.item()) == 0 and int(err2.item()) == 0
        for k in ("lat_k", "lat_v", "sk", "sv", "lens"):
            assert torch.equal(st[k], two[k]), (name, k)
        assert torch.equal(out1, out2), name

    # and the oracle's append + decode
    lk, sk, lv, sv, nl, _, _, _ = O.latent_append(ai.x[0], ai.A_k, ai.A_v, d.seq_lens, d.lat_k, d.scale_k, d.lat_v,
                                                  d.scale_v, w.r, w.bits, w.hadamard_block)
    ref = O.wsvd_decode(d.q, lk, sk, lv, sv, d.Bk, d.Bv, nl, w.r, w.bits)
    assert np.array_equal(one["lens"].cpu().numpy(), np.asarray(lens0) + 1)
    assert_attention_close(out1.cpu().numpy(), ref, f"step {name}")


ONE_KERNEL = ("llava7b", "llava7b-chunk-start", "llava7b-middle", "llava7b-chunk-end", "llava7b-first-row",
              "int4-one-kernel", "two-rank", "one-rank")


def test_step_launch_count_matches_the_path():
    """One kernel for the single-sequence cluster-path cases, the append plus
    the decode's launches otherwise."""
    lc = W.wsvd_step_launch_count
    for name, (w, _) in CASES.items():
        n = lc(w.B, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap, w.hadamard_block)
        dn = W.wsvd_decode_launch_count(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap)
        assert n == (1 if name in ONE_KERNEL else 1 + dn), name
    w = WL.LLAVA7B
    assert lc(w.B, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap, w.hadamard_block, w8=True) == 1
    assert lc(2, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap, w.hadamard_block) == 2  # two sequences: append + decode
    assert lc(1, w.H, w.Hd, w.E, 16, w.bits, w.L_cap, w.hadamard_block) == 2  # two tokens per lane and tile
    assert lc(0, w.H, w.Hd, w.E, w.r, w.bits, w.L_cap, w.hadamard_block) == 0


@pytest.mark.parametrize("start", ["full", "negative"])
def test_step_with_no_free_row_equals_the_two_calls(start):
    """A full cache (length L_cap) or an invalid length: nothing is appended,
    the error bits and the output are those of the two calls."""
    w = WL.LLAVA7B
    d, ai = _inputs(w, [w.L_cap - 1], seed=5)
    d.seq_lens[:] = w.L_cap if start == "full" else -3
    x = q_tensor(ai.x_bits[0], "bf16")
    A_k, A_v, B_k, B_v = dev(ai.A_k), dev(ai.A_v), dev(d.Bk), dev(d.Bv)
    q = q_tensor(d.q_bits, w.q_dtype)
    two, one = _device_state(d), _device_state(d)
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    err1 = torch.zeros(1, dtype=torch.int32, device="cuda")
    W.wsvd_latent_append(x, A_k, A_v, two["lens"], two["lat_k"], two["lat_v"], two["sk"], two["sv"], bits=w.bits,
                         err=err2)
    out2 = W.wsvd_decode_attention(q, two["lat_k"], two["lat_v"], two["sk"], two["sv"], B_k, B_v, two["lens"],
                                   bits=w.bits, err=err2)
    out1 = W.wsvd_append_and_decode(x, A_k, A_v, one["lens"], one["lat_k"], one["lat_v"], one["sk"], one["sv"], q,
                                    B_k, B_v, bits=w.bits, err=err1)
    torch.cuda.synchronize()
    assert int(err1.item()) == int(err2.item()) != 0
    for k in ("lat_k", "lat_v", "sk", "sv", "lens"):
        assert torch.equal(one[k], two[k]), k
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("name", ["llava7b", "llava7b-chunk-start", "int4-one-kernel"])
def test_step_ignores_rows_at_and_past_the_new_one(name):
    """Rows from the new token's position on (the row the append writes, and
    the cache's unused tail) hold random bytes: the step's output and the
    rows it writes are those of a clean cache, bit for bit, and every byte
    past the new row is left as it was."""
    w, lens0 = CASES[name]
    d, ai = _inputs(w, lens0, seed=41)
    x = q_tensor(ai.x_bits[0], "bf16")
    A_k, A_v, B_k, B_v = dev(ai.A_k), dev(ai.A_v), dev(d.Bk), dev(d.Bv)
    q = q_tensor(d.q_bits, w.q_dtype)
    clean = _device_state(d)
    g = np.random.default_rng(7)
    for b, n in enumerate(lens0):
        for a in (d.lat_k, d.lat_v):
            a[b, :, n:] = g.integers(0, 256, size=a[b, :, n:].shape, dtype=np.uint8)
        for a in (d.scale_k, d.scale_v):
            a[b, :, n:] = g.standard_normal(a[b, :, n:].shape).astype(np.float16) * 1e4
    dirty = _device_state(d)
    outs = [W.wsvd_append_and_decode(x, A_k, A_v, st["lens"], st["lat_k"], st["lat_v"], st["sk"], st["sv"], q, B_k,
                                     B_v, bits=w.bits, hadamard_block=w.hadamard_block) for st in (clean, dirty)]
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]), name
    for k in ("lat_k", "lat_v", "sk", "sv"):
        for b, n in enumerate(lens0):
            assert torch.equal(clean[k][b, :, :n + 1], dirty[k][b, :, :n + 1]), (name, k)
    after = _device_state(d)  # the poisoned inputs, untouched
    for k in ("lat_k", "lat_v", "sk", "sv"):
        for b, n in enumerate(lens0):
            assert torch.equal(dirty[k][b, :, n + 1:], after[k][b, :, n + 1:]), (name, k)


def test_step_validates_before_launching():
    w, lens0 = CASES["llava7b"]
    d, ai = _inputs(w, lens0, seed=3)
    st = _device_state(d)
    x = q_tensor(ai.x_bits[0], "bf16")
    q = q_tensor(d.q_bits, w.q_dtype)
    bad_B_v = dev(d.Bv)[:, :, :64].contiguous()  # wrong head dim: rejected by the binding
    with pytest.raises(W.WsvdError):
        W.wsvd_append_and_decode(x, dev(ai.A_k), dev(ai.A_v), st["lens"], st["lat_k"], st["lat_v"], st["sk"],
                                 st["sv"], q, dev(d.Bk), bad_B_v, bits=w.bits)
    # a decode-side failure in the library (too small a decode workspace) leaves the cache untouched
    small = W.workspace(16)
    with pytest.raises(W.WsvdError):
        W.wsvd_append_and_decode(x, dev(ai.A_k), dev(ai.A_v), st["lens"], st["lat_k"], st["lat_v"], st["sk"],
                                 st["sv"], q, dev(d.Bk), dev(d.Bv), bits=w.bits, decode_ws=small)
    torch.cuda.synchronize()
    assert np.array_equal(st["lens"].cpu().numpy(), np.asarray(lens0))
    assert torch.equal(st["lat_k"], dev(d.lat_k))


def test_decode_launch_count_matches_the_path():
    """One kernel for the cluster path (the LLaVA layer), two for the split-L
    grid behind its q' projection (long contexts, ragged batches)."""
    lc = W.wsvd_decode_launch_count
    w = WL.LLAVA7B
    assert lc(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap) == 1
    for w in (WL.LONG[16], WL.LONG[32], WL.LONG[64], WL.RAGGED, WL.CMP[8192]):
        assert lc(w.B, w.H, w.Hd, w.r, w.bits, w.L_cap) == 2, w.name


@pytest.mark.parametrize("name,memory", [("llava7b", "pinned"), ("llava7b", "pinned-one-buffer"),
                                         ("llava7b", "pinned-direct"), ("llava7b", "pageable"), ("long-r32", "pinned"),
                                         ("ragged-int4", "pinned"), ("ragged-int4", "pinned-direct"),
                                         ("int4-one-kernel", "pinned"), ("int4-one-kernel", "pinned-direct")])
def test_step_from_host_buffers_equals_device_step(name, memory):
    """wsvd_append_and_decode_host gives bit for bit what wsvd_append_and_decode
    gives on the same values already on the device, on two steps in a row
    whose host inputs differ (the second step's values are written into the
    same host buffers).  Pinned buffers are read and written by the kernels in
    place (replayed from one captured graph, or one direct call per step);
    pageable ones go through copies."""
    w, lens0 = CASES[name]
    lens0 = [min(n, w.L_cap - 2) for n in lens0]  # two steps in a row: room for two appended rows
    d, ai = _inputs(w, lens0, seed=33)
    ai2 = WL.append_inputs(w, seed=34, steps=1)
    q2_bits = WL.decode_inputs(w, seed=35, lens=np.asarray(lens0) + 1).q_bits
    qdt = torch.float16 if w.q_dtype == "fp16" else torch.bfloat16
    xs = [torch.from_numpy(a.x_bits[0].view(np.int16).copy()) for a in (ai, ai2)]
    qs = [torch.from_numpy(b.view(np.int16).copy()) for b in (d.q_bits, q2_bits)]
    xb, qb = xs[0], qs[0]
    if memory == "pinned-one-buffer":
        io = torch.cat([xb.reshape(-1), qb.reshape(-1)]).pin_memory()
        x_host = io[:xb.numel()].view(torch.bfloat16).view(xb.shape)
        q_host = io[xb.numel():].view(qdt).view(qb.shape)
    elif memory in ("pinned", "pinned-direct"):
        x_host = xb.view(torch.bfloat16).pin_memory()
        q_host = qb.view(qdt).pin_memory()
    else:
        x_host = xb.view(torch.bfloat16).clone()
        q_host = qb.view(qdt).clone()
    out_host = torch.full((w.B, w.H, w.Hd), float("nan"), dtype=torch.float32)
    if memory != "pageable":
        out_host = out_host.pin_memory()
    assert x_host.is_pinned() == (memory != "pageable") and out_host.is_pinned() == (memory != "pageable")
    A_k, A_v, B_k, B_v = dev(ai.A_k), dev(ai.A_v), dev(d.Bk), dev(d.Bv)
    dv, hs = _device_state(d), _device_state(d)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    step = W.StepFromHost(x_host, A_k, A_v, hs["lens"], hs["lat_k"], hs["lat_v"], hs["sk"], hs["sv"], q_host, B_k,
                          B_v, out_host, bits=w.bits, hadamard_block=w.hadamard_block, err=err,
                          graph=False if memory == "pinned-direct" else None)
    assert step.uses_graph == (memory in ("pinned", "pinned-one-buffer"))
    for rep in range(2):
        x_host.view(torch.int16).copy_(xs[rep].view(x_host.shape))
        q_host.view(torch.int16).copy_(qs[rep].view(q_host.shape))
        out_dev = W.wsvd_append_and_decode(x_host.cuda(), A_k, A_v, dv["lens"], dv["lat_k"], dv["lat_v"], dv["sk"],
                                           dv["sv"], q_host.cuda(), B_k, B_v, bits=w.bits,
                                           hadamard_block=w.hadamard_block)
        torch.cuda.synchronize()
        step()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(out_host, out_dev.cpu()), (name, memory, rep)
        for k in ("lat_k", "lat_v", "sk", "sv", "lens"):
            assert torch.equal(hs[k], dv[k]), (name, memory, k, rep)
    assert np.array_equal(hs["lens"].cpu().numpy(), np.asarray(lens0) + 2)
