"""The C-ABI library loads on a host without a GPU, exports every symbol the
public header declares, and its host-only entry points (sizes, validation)
behave as documented.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import oracle as O
import rank_kv_cache_wsvd_b200 as W
from rank_kv_cache_wsvd_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wsvd.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\**([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from rank_kv_cache_wsvd_b200 import build
        build.build()
    return _lib.load()


def test_header_symbols_are_exported_and_bound(lib):
    names = _declared_functions()
    assert len(names) >= 12, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in wsvd.h but not exported"
        assert n in _lib.SIGNATURES, f"{n} has no Python binding signature"
    assert set(_lib.SIGNATURES) == set(names)


def test_status_strings_and_version(lib):
    assert lib.wsvd_abi_version() == 100
    assert lib.wsvd_status_string(0) == b"ok"
    assert lib.wsvd_status_string(4) == b"workspace too small"
    assert lib.wsvd_status_string(99) == b"unknown status"


@pytest.mark.parametrize("B,H,L,r,bits", [(1, 4, 256, 16, 8), (16, 32, 4096, 32, 4), (4, 32, 32768, 64, 8)])
def test_cache_byte_counts_match_oracle(lib, B, H, L, r, bits):
    assert W.wsvd_cache_bytes(B, H, L, r, bits) == O.wsvd_cache_bytes(B, H, L, r, bits)
    assert W.shared_cache_bytes(B, L, 512) == O.shared_cache_bytes(B, L, 512)
    assert W.dense_cache_bytes(B, H, L, 128) == O.dense_cache_bytes(B, H, L, 128)


def test_workspace_sizes_hold_only_partials(lib):
    """The decode workspace holds split partials (W + 2 floats per slot), one
    counter per head and the projected queries q' (W floats per head), never
    an L x Hd buffer: reconstructed K/V are not materialised."""
    B, H, r, L = 4, 32, 32, 32768
    a16 = lambda v: (v + 15) // 16 * 16
    size = lambda W_: a16((2048 + B * H) * (W_ + 2) * 4) + a16(B * H * 4) + a16(B * H * W_ * 4)
    ws = W.wsvd_decode_workspace_size(B, H, r)
    assert ws == size(r)
    assert ws < B * H * L * 128 * 2 / 100  # far below one reconstructed K
    assert W.dense_decode_workspace_size(B, H, 128) == size(128)
    assert W.shared_decode_workspace_size(B, H, 512) == size(512)
    assert W.wsvd_append_workspace_size() == 256


def test_host_validation_rejects_before_launch(lib):
    p = ctypes.c_void_p(16)  # never dereferenced: validation fails first
    # null seq_lens
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 8, 256, None, p, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                     None, None) == 1
    # bits not in {4, 8}
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 6, 256, p, p, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                     None, None) == 1
    # row bytes not a multiple of 16 (r = 16, int4 -> 8 bytes)
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 4, 256, p, p, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                     None, None) == 2
    # L_cap not a multiple of 8
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 8, 257, p, p, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                     None, None) == 2
    # misaligned pointer
    bad = ctypes.c_void_p(24)
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 8, 256, p, bad, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                     None, None) == 1
    # workspace too small
    assert lib.wsvd_decode_attention(1, 4, 64, 16, 8, 256, p, p, 0, p, p, p, p, p, p, 0.0, p, p, 64,
                                     None, None) == 4
    # int8 weights: the B scales are staged by bulk copies and must be 16-byte aligned
    assert lib.wsvd_decode_attention_w8(1, 4, 64, 16, 8, 256, p, p, 0, p, p, p, p, p, p, bad, p, 0.0, p, p, 1 << 20,
                                        None, None) == 1
    assert lib.wsvd_decode_attention_w8(1, 4, 64, 16, 8, 256, p, p, 0, p, p, p, p, p, p, p, bad, 0.0, p, p, 1 << 20,
                                        None, None) == 1
    # empty batch is a no-op
    assert lib.wsvd_decode_attention(0, 4, 64, 16, 8, 256, None, None, 0, None, None, None, None, None, None,
                                     0.0, None, None, 0, None, None) == 0
    # append: hadamard block not a power of two / E not a multiple of it / B too large
    assert lib.wsvd_latent_append(1, 4, 256, 16, 8, 8, 96, p, 1, p, p, p, p, p, p, p, p, 256, None, None) == 1
    assert lib.wsvd_latent_append(1, 4, 200, 16, 8, 8, 128, p, 1, p, p, p, p, p, p, p, p, 256, None, None) == 1
    assert lib.wsvd_latent_append(17, 4, 256, 16, 8, 8, 128, p, 1, p, p, p, p, p, p, p, p, 256, None, None) == 2
    # r / 8 column groups must divide a warp: r = 24 or 40 is rejected
    for r in (24, 40):
        assert lib.wsvd_latent_append(1, 4, 256, r, 8, 8, 128, p, 1, p, p, p, p, p, p, p, p, 256, None, None) == 2
    assert lib.wsvd_latent_append(1, 4, 256, 16, 8, 8, 128, p, 1, p, p, p, p, p, p, p, p, 8, None, None) == 4
    # dense / shared: unsupported widths
    assert lib.dense_decode_attention(1, 4, 48, 256, p, p, 0, p, p, 0.0, p, p, 1 << 22, None, None) == 2
    assert lib.shared_latent_svd_decode(1, 4, 128, 384, 256, p, p, 0, p, p, p, p, 0.0, p, p, 1 << 24,
                                        None, None) == 2


def test_decode_launch_count_rejects_bad_sizes(lib):
    """wsvd_decode_launch_count answers 0 for sizes the decode would reject."""
    assert W.wsvd_decode_launch_count(0, 32, 128, 32, 8, 1600) == 0
    assert W.wsvd_decode_launch_count(1, 32, 128, 32, 5, 1600) == 0
    assert W.wsvd_decode_launch_count(1, 32, 128, 3, 4, 1600) == 0  # r * bits not a whole byte
    assert W.wsvd_decode_launch_count(1, 32, 128, 24, 8, 1600) == 0  # 24-byte rows are not instantiated


def test_step_launch_count_rejects_bad_sizes(lib):
    """wsvd_step_launch_count answers 0 for sizes the step would reject."""
    assert W.wsvd_step_launch_count(0, 32, 128, 4096, 32, 8, 1600) == 0
    assert W.wsvd_step_launch_count(1, 32, 128, 4096, 32, 5, 1600) == 0
    assert W.wsvd_step_launch_count(1, 32, 128, 4096, 32, 8, 1600, hadamard_block=96) == 0  # not a power of two
    assert W.wsvd_step_launch_count(1, 32, 128, 4000, 32, 8, 1600) == 0  # E not a multiple of the block
    assert W.wsvd_step_launch_count(1, 32, 128, 4096, 24, 8, 1600) == 0  # 24-byte rows are not instantiated


def test_prefill_workspace_and_host_validation(lib):
    """The prefill scratch holds the split rotated activations (two fp16 copies
    of the B x T x E block) and one power-of-two scale per token row; bad
    shapes are refused before anything is launched."""
    a16 = lambda v: (v + 15) // 16 * 16
    assert W.wsvd_prefill_workspace_size(1, 576, 4096) == 2 * a16(576 * 4096 * 2) + a16(576 * 4)
    assert W.wsvd_prefill_workspace_size(0, 576, 4096) == 0
    p = ctypes.c_void_p(16)
    ws = W.wsvd_prefill_workspace_size(2, 3, 256)
    args = lambda B=2, T=3, H=4, E=256, r=16, bits=8, L=64, blk=128, ptr=p, nbytes=ws: (
        B, T, H, E, r, bits, L, blk, ptr, 1, p, p, p, p, p, p, p, p, nbytes, None, None)
    assert lib.wsvd_latent_prefill(*args(blk=96)) == 1            # block not a power of two
    assert lib.wsvd_latent_prefill(*args(bits=6)) == 1            # bits not in {4, 8}
    assert lib.wsvd_latent_prefill(*args(r=24)) == 2              # r must divide the 128-column tile
    assert lib.wsvd_latent_prefill(*args(E=272, blk=16)) == 2     # E not a multiple of the 64-wide k tile
    assert lib.wsvd_latent_prefill(*args(E=32768)) == 2           # row does not fit the rotation's shared memory
    assert lib.wsvd_latent_prefill(*args(ptr=ctypes.c_void_p(24))) == 1  # misaligned x
    assert lib.wsvd_latent_prefill(*args(ptr=None)) == 1          # null x
    assert lib.wsvd_latent_prefill(*args(nbytes=ws - 16)) == 4    # workspace too small
    assert lib.wsvd_latent_prefill(*args(T=0, ptr=None)) == 0     # empty block: nothing launched
    assert lib.wsvd_latent_prefill(*args(B=0, ptr=None)) == 0
    assert lib.wsvd_latent_prefill(*args(T=-1)) == 1


def test_noalloc_checks_come_first_and_match_the_workspace_entry_point(lib):
    """The no-allocation decode answers the first argument checks exactly as
    wsvd_decode_attention does, before any CUDA call (so on this host too)."""
    p = ctypes.c_void_p(16)
    for B, H, L_cap, want in [(0, 0, 64, 1), (-1, 4, 64, 1), (1, 4, -8, 1), (0, 4, 64, 0)]:
        ws = lib.wsvd_decode_attention(B, H, 64, 16, 8, L_cap, p, p, 0, p, p, p, p, p, p, 0.0, p, p, 1 << 20,
                                       None, None)
        na = lib.wsvd_decode_attention_noalloc(B, H, 64, 16, 8, L_cap, p, p, 0, p, p, p, p, p, p, 0.0, p, None,
                                               None)
        assert ws == na == want, (B, H, L_cap, ws, na)


def test_fold_rejects_overlapping_outputs(lib):
    """Outputs may share no byte with any input or with each other: exact
    aliasing, a partial overlap and two overlapping outputs are refused before
    any launch."""
    H, E, r, Hd = 2, 64, 16, 64
    na, nb, ns = H * E * r * 2, H * r * Hd * 2, H * r * r * 4
    base = 1 << 20
    S2k, S2v = base, base + ns
    Ak, Av = base + 2 * ns, base + 2 * ns + na
    Bk, Bv = Av + na, Av + na + nb
    free = Bv + nb + 4096
    outs = [free, free + na, free + 2 * na, free + 2 * na + nb]

    def call(o):
        return lib.wsvd_fold_latent_rotation(H, E, r, Hd, *[ctypes.c_void_p(v) for v in
                                                             (S2k, S2v, Ak, Av, Bk, Bv, *o)], None)
    assert call([Ak, outs[1], outs[2], outs[3]]) == 1              # A_k_out is A_k
    assert call([outs[0], Av + 16, outs[2], outs[3]]) == 1         # A_v_out starts inside A_v
    assert call([outs[0], outs[1], S2v + ns - 16, outs[3]]) == 1   # B_k_out runs into S2_v's tail
    assert call([outs[0], outs[0] + 16, outs[2], outs[3]]) == 1    # two outputs overlap


def test_step_from_host_validation(lib):
    """wsvd_append_and_decode_host refuses null host buffers and a small step
    workspace before anything is queued; its workspace holds the append and
    decode workspaces plus device copies of x, q and out."""
    B, H, Hd, E, r = 1, 4, 64, 256, 16
    a16 = lambda v: (v + 15) // 16 * 16
    need = W.wsvd_step_host_workspace_size(B, H, Hd, E, r)
    assert need == 256 + W.wsvd_decode_workspace_size(B, H, r) + a16(B * E * 2) + a16(B * H * Hd * 2) + \
        a16(B * H * Hd * 4)
    p = ctypes.c_void_p(16)
    args = lambda xh=p, nbytes=need: (B, H, Hd, E, r, 8, 64, 128, xh, 1, p, p, p, p, p, p, p, p, 0, p, p, 0.0, p, p,
                                      nbytes, None, None)
    assert lib.wsvd_append_and_decode_host(*args(xh=None)) == 1
    assert lib.wsvd_append_and_decode_host(*args(nbytes=need - 16)) == 4


def test_step_graph_needs_pinned_buffers_and_a_handle(lib):
    """The captured host-buffer step refuses host pointers that are not pinned
    and mapped (WSVD_ERR_UNSUPPORTED, handle set to NULL) and a missing handle
    slot; a NULL handle is refused by launch and ignored by destroy."""
    B, H, Hd, E, r = 1, 4, 64, 256, 16
    need = W.wsvd_step_host_workspace_size(B, H, Hd, E, r)
    p = ctypes.c_void_p(16)
    args = (B, H, Hd, E, r, 8, 64, 128, p, 1, p, p, p, p, p, p, p, p, 0, p, p, 0.0, p, p, need, None)
    h = ctypes.c_void_p(1234)
    assert lib.wsvd_step_host_graph_create(*args, ctypes.byref(h)) == 2
    assert h.value is None
    assert lib.wsvd_step_host_graph_create(*args, None) == 1
    assert lib.wsvd_step_host_graph_launch(None, None) == 1
    lib.wsvd_step_host_graph_destroy(None)


def test_grouped_decode_workspace_and_validation(lib):
    """Grouped / multi-token decode: the workspace holds split partials (at most
    64 splits of 128-token tiles) of up to 16 queries per (sequence, latent
    head, query chunk) and one counter per chunk; unsupported shapes are
    refused before anything is launched."""
    a16 = lambda v: (v + 15) // 16 * 16
    B, Tq, Hq, Hkv, r, L = 2, 4, 32, 8, 32, 1600
    nq, nqc, slots = 16, 1, 13  # G * Tq = 16 queries; ceil(1600 / 128) = 13 tiles
    qblock = 48 * 32 + 16 * 4    # q' planes of a group: 3 x 16 rows of 32 bytes, then 16 steps
    want = a16(B * Hkv * nqc * slots * nq * (r + 2) * 4) + a16(B * Hkv * nqc * 4) + a16(B * Hkv * nqc * qblock)
    assert W.wsvd_decode_multi_workspace_size(B, Tq, Hq, Hkv, r, L) == want
    assert lib.wsvd_decode_gqa_workspace_size(B, Hq, Hkv, r, L) == W.wsvd_decode_multi_workspace_size(
        B, 1, Hq, Hkv, r, L)
    # G * Tq = 32 queries: two chunks of 16; 64-split cap at 32768 tokens
    assert W.wsvd_decode_multi_workspace_size(1, 4, 32, 4, 32, 32768) == \
        a16(1 * 4 * 2 * 64 * 16 * 34 * 4) + a16(1 * 4 * 2 * 4) + a16(1 * 4 * 2 * qblock)
    p = ctypes.c_void_p(16)
    ws = 1 << 24
    args = lambda B=1, Tq=1, Hq=8, Hkv=2, Hd=64, r=32, bits=8, L=64, qp=p: (
        B, Tq, Hq, Hkv, Hd, r, bits, L, p, qp, 0, p, p, p, p, p, p, 0.0, p, p, ws, None, None)
    assert lib.wsvd_decode_multi(*args(Hq=6, Hkv=4)) == 1      # Hq not a multiple of Hkv
    assert lib.wsvd_decode_multi(*args(Tq=9, Hq=16, Hkv=2)) == 2  # G * Tq = 72 > 64
    assert lib.wsvd_decode_multi(*args(r=8)) == 2               # 8-byte rows
    assert lib.wsvd_decode_multi(*args(Hd=48)) == 2
    assert lib.wsvd_decode_multi(*args(L=60)) == 2              # L_cap not a multiple of 8
    assert lib.wsvd_decode_multi(*args(bits=6)) == 1
    assert lib.wsvd_decode_multi(*args(qp=None)) == 1
    assert lib.wsvd_decode_multi(*args(qp=ctypes.c_void_p(24))) == 1
    assert lib.wsvd_decode_multi(*args(B=0, qp=None)) == 0
    small = list(args())
    small[20] = 16
    assert lib.wsvd_decode_multi(*small) == 4
