"""The C ABI (include/s3r.h) on the host: the library loads, exports every declared entry point,
and rejects bad arguments with the documented status before touching the device.

None of these tests launches a kernel: every call below fails host-side validation first, so
they run without a GPU.
"""
import ctypes
import os
import re

import pytest

from sparse_global_attention_s3r_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "s3r.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(s3r_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) == 17, names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.EXPORTS)


def test_status_strings_and_version():
    assert _lib.status_string(0) == "S3R_OK"
    assert _lib.status_string(5) == "S3R_ERR_TIMEOUT"
    assert _lib.status_string(99) == "S3R_ERR_UNKNOWN"
    assert _lib.load().s3r_version() >= 100


def _params(**kw):
    base = dict(L=1024, H=2, d=64, block=64, qblock=64, topk=4, scale=0.0, flags=0, dev_status=None)
    base.update(kw)
    return _lib.Params(**base)


# fake, never-dereferenced device addresses: validation must reject before any use
A16 = ctypes.c_void_p(1 << 20)
A8 = ctypes.c_void_p((1 << 20) + 8)
A256 = ctypes.c_void_p(1 << 24)
A16_NOT256 = ctypes.c_void_p((1 << 20) + 16)


@pytest.mark.parametrize("kw,want", [
    (dict(d=128), _lib.S3R_ERR_UNSUPPORTED),
    (dict(d=32), _lib.S3R_ERR_UNSUPPORTED),
    (dict(block=16), _lib.S3R_ERR_UNSUPPORTED),
    (dict(block=256), _lib.S3R_ERR_UNSUPPORTED),
    (dict(qblock=128), _lib.S3R_ERR_UNSUPPORTED),
    (dict(L=0), _lib.S3R_ERR_INVALID_ARG),
    (dict(H=0), _lib.S3R_ERR_INVALID_ARG),
    (dict(topk=0), _lib.S3R_ERR_INVALID_ARG),
    (dict(topk=17), _lib.S3R_ERR_INVALID_ARG),  # nb = 16
    (dict(topk=4, forced=13), _lib.S3R_ERR_INVALID_ARG),  # forced + topk > nb
    (dict(forced=-1), _lib.S3R_ERR_INVALID_ARG),
    # 2-D windows: L must be whole views, win_h must divide b, special must fit one block
    (dict(L=1001, grid_h=3, grid_w=3, special=1, win_h=2), _lib.S3R_ERR_INVALID_ARG),
    (dict(L=1020, grid_h=10, grid_w=10, special=2, win_h=3), _lib.S3R_ERR_INVALID_ARG),
    (dict(L=6 * 166, block=32, grid_h=10, grid_w=10, special=66, win_h=4), _lib.S3R_ERR_INVALID_ARG),
    (dict(L=1020, grid_h=10, grid_w=-1, special=2, win_h=2), _lib.S3R_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.S3R_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.S3R_ERR_INVALID_ARG),
    (dict(L=_lib.S3R_MAX_BLOCKS * 32 + 1, block=32, topk=1), _lib.S3R_ERR_UNSUPPORTED),
])
def test_bad_sizes_are_rejected_by_every_entry_point(kw, want):
    lib = _lib.load()
    p = ctypes.byref(_params(**kw))
    s = None
    assert lib.s3r_compress_kv(p, A16, A16, A16, A16, s) == want
    assert lib.s3r_cmp_attn_and_score(p, A16, A16, A16, A16, A16, A16, s) == want
    assert lib.s3r_topk_blocks(p, A16, A16, s) == want
    assert lib.s3r_sel_attn(p, A16, A16, A16, A16, A16, s) == want
    assert lib.s3r_gate_combine(p, A16, A16, A16, A16, s) == want
    assert lib.s3r_sparse_attn_fwd(p, A16, A16, A16, A16, A16, None, A256, 1 << 40, s) == want
    assert lib.s3r_sparse_attn_bwd(p, *[A16] * 10, A256, 1 << 40, s) == want
    assert lib.s3r_workspace_bytes(p) == 0
    assert lib.s3r_bwd_workspace_bytes(p) == 0


def test_null_and_misaligned_pointers_are_rejected():
    lib = _lib.load()
    p = ctypes.byref(_params())
    for bad in (None, A8):
        assert lib.s3r_compress_kv(p, bad, A16, A16, A16, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_compress_kv(p, A16, A16, A16, bad, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_cmp_attn_and_score(p, A16, A16, A16, A16, A16, bad, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_topk_blocks(p, bad, A16, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_sel_attn(p, A16, A16, A16, bad, A16, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_gate_combine(p, A16, A16, bad, A16, None) == _lib.S3R_ERR_INVALID_ARG
        assert lib.s3r_sparse_attn_fwd(p, A16, bad, A16, A16, A16, None, A256, 1 << 40, None) == _lib.S3R_ERR_INVALID_ARG
    for i in range(10):  # every array of the backward is required and 16-byte aligned
        for bad in (None, A8):
            args = [A16] * 10
            args[i] = bad
            assert lib.s3r_sparse_attn_bwd(p, *args, A256, 1 << 40, None) == _lib.S3R_ERR_INVALID_ARG
    # idx_out is optional but must be aligned when given
    assert lib.s3r_sparse_attn_fwd(p, A16, A16, A16, A16, A16, A8, A256, 1 << 40, None) == _lib.S3R_ERR_INVALID_ARG
    # a misaligned status word
    p2 = ctypes.byref(_params(dev_status=(1 << 20) + 2))
    assert lib.s3r_topk_blocks(p2, A16, A16, None) == _lib.S3R_ERR_INVALID_ARG
    assert lib.s3r_read_device_status(None, None, A16) == _lib.S3R_ERR_INVALID_ARG
    assert lib.s3r_topk_blocks(None, A16, A16, None) == _lib.S3R_ERR_INVALID_ARG


def test_workspace_checks():
    lib = _lib.load()
    prm = _params()
    need = lib.s3r_workspace_bytes(ctypes.byref(prm))
    p = ctypes.byref(prm)
    assert lib.s3r_sparse_attn_fwd(p, A16, A16, A16, A16, A16, None, None, need, None) == _lib.S3R_ERR_WORKSPACE
    assert lib.s3r_sparse_attn_fwd(p, A16, A16, A16, A16, A16, None, A256, need - 1, None) == _lib.S3R_ERR_WORKSPACE
    assert lib.s3r_sparse_attn_fwd(p, A16, A16, A16, A16, A16, None, A16_NOT256, need, None) == _lib.S3R_ERR_WORKSPACE
    assert lib.s3r_workspace_status_word(A256) == A256.value
    need = lib.s3r_bwd_workspace_bytes(ctypes.byref(prm))
    for ws, n in ((None, need), (A256, need - 1), (A16_NOT256, need)):
        assert lib.s3r_sparse_attn_bwd(p, *[A16] * 10, ws, n, None) == _lib.S3R_ERR_WORKSPACE


def kv_chunks(L, H, b):
    """Pieces of the dKc/dVc kernel's walk over the queries: the smallest c <= 16 (pieces of at
    least 32 64-query steps) whose CTAs fill the waves of 148 SMs x 2 resident CTAs to 95 %, else
    the best-filling c; then as many pieces as ceil(steps / ceil(steps / c))."""
    nb = -(-L // b)
    tiles, steps, res = -(-nb // 128) * H, -(-L // 64), 2 * 148
    best, best_fill = 1, 0.0
    for c in range(1, 17):
        if c > 1 and -(-steps // c) < 32:
            break
        ctas = c * tiles
        fill = ctas / (-(-ctas // res) * res)
        if 100 * ctas >= 95 * (-(-ctas // res) * res):
            best = c
            break
        if fill > best_fill:
            best, best_fill = c, fill
    per = -(-steps // best)
    return -(-steps // per)


def test_kv_chunks_at_the_workload_sizes():
    # 1000 views: 2688 CTAs fill 9.08 waves, 18.16 in two pieces; 100 views: 272 CTAs
    assert kv_chunks(1374000, 16, 64) == 2
    assert kv_chunks(137400, 16, 64) == 13
    assert kv_chunks(1, 2, 32) == 1
    assert kv_chunks(40000, 1, 64) == 16  # the backward parity case of the most pieces


@pytest.mark.parametrize("L,H,b,k,F", [(1024, 2, 64, 4, 0), (1374000, 16, 64, 32, 0),
                                       (43968, 16, 64, 16, 22), (1, 1, 128, 1, 0)])
def test_bwd_workspace_size_matches_layout(L, H, b, k, F):
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=F)
    nb, nqb, d = cfg.nb, cfg.nqb, 64
    Lp = (L + 127) // 128 * 128
    want = (r256(4) + 2 * r256(nb * H * d * 2) + 2 * r256(nb * b * H * d * 2)
            + 2 * r256(L * H * d * 4) + 2 * r256(H * L * 4) + r256(6 * H * Lp * 4)
            + 2 * r256(nb * H * d * 4) + 2 * r256(H * nb * 4) + r256(H * (nb + 1) * 4)
            + r256(H * nqb * (F + k) * 4) + r256(H * nb * max(1, b // 64) * 4)
            + 2 * r256((nqb + 1) * 4) + r256((nqb + 2) * 4))
    c = kv_chunks(L, H, b)
    if c > 1:  # the pieces' partial dKc, dVc
        want += r256(2 * c * nb * H * d * 4)
    assert api.bwd_workspace_bytes(cfg) == want


@pytest.mark.parametrize("L,H,b,k", [(1024, 2, 64, 4), (1374000, 16, 64, 32), (3000, 2, 32, 40)])
def test_save_for_backward_workspaces(L, H, b, k):
    """With S3R_FLAG_SAVE_FOR_BWD the forward's workspace adds O_sel and both lse, and the
    backward's workspace is the forward's followed by the backward's own scratch."""
    import dataclasses

    cfg = api.Config(L=L, H=H, block=b, topk=k)
    save = dataclasses.replace(cfg, save_for_backward=True)
    fwd, fwd_s = api.workspace_bytes(cfg), api.workspace_bytes(save)
    assert fwd_s == fwd + r256(L * H * 64 * 4) + 2 * r256(H * L * 4)
    nb, nqb = cfg.nb, cfg.nqb
    Lp = (L + 127) // 128 * 128
    scratch = (r256(6 * H * Lp * 4) + 2 * r256(nb * H * 64 * 4) + 2 * r256(H * nb * 4)
               + r256(H * (nb + 1) * 4) + r256(H * nqb * k * 4) + r256(H * nb * max(1, b // 64) * 4)
               + 2 * r256((nqb + 1) * 4) + r256((nqb + 2) * 4))
    c = kv_chunks(L, H, b)
    if c > 1:
        scratch += r256(2 * c * nb * H * 64 * 4)
    assert api.bwd_workspace_bytes(save) == fwd_s + scratch
    lib = _lib.load()
    p = ctypes.byref(save.params())
    assert lib.s3r_sparse_attn_bwd(p, *[A16] * 10, A256, fwd_s, None) == _lib.S3R_ERR_WORKSPACE


def test_save_for_backward_needs_the_slot_copies():
    """The saving forward keeps the slot-order K/V copies for the backward: sizes whose copies
    exceed 32-bit row coordinates are rejected before any launch."""
    lib = _lib.load()
    big = _params(L=65536, H=65535, block=64, topk=1, flags=_lib.S3R_FLAG_SAVE_FOR_BWD)
    assert lib.s3r_sparse_attn_fwd(ctypes.byref(big), A16, A16, A16, A16, A16, None, A256,
                                   1 << 62, None) == _lib.S3R_ERR_UNSUPPORTED


def test_bwd_rejects_slot_copies_beyond_32_bit_rows():
    lib = _lib.load()
    big = _params(L=65536, H=65535, block=64, topk=1)  # H * nb * b = 65535 * 65536 > 2^31 - 1
    assert lib.s3r_sparse_attn_bwd(ctypes.byref(big), *[A16] * 10, A256, 1 << 62,
                                   None) == _lib.S3R_ERR_UNSUPPORTED


def r256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("L,H,b,k,F", [(1024, 2, 64, 4, 0), (1374000, 16, 64, 32, 0),
                                       (274800, 16, 32, 8588, 0), (1, 1, 128, 1, 0),
                                       (43968, 16, 64, 16, 22), (43968, 16, 64, 40, 22)])
def test_workspace_size_matches_layout(L, H, b, k, F):
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=F)
    nb, nqb, d = cfg.nb, cfg.nqb, 64
    scores = H * nqb * nb * 4 if k > 32 else 0  # materialised only when k exceeds 32
    copies = 2 * r256(nb * b * H * d * 2) if H * nb * b <= 2**31 - 1 else 0  # head-major K, V
    want = (r256(4) + 2 * r256(nb * H * d * 2) + copies + r256(L * H * d * 4)
            + r256(scores) + r256(H * nqb * (F + k) * 4))
    assert api.workspace_bytes(cfg) == want


def test_compute_calls_need_cuda_tensors():
    cfg = api.Config(L=64, H=1, block=64, topk=1)
    import torch

    k = torch.zeros(64, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.compress_kv(cfg, k, k)


def test_static_entry_point_rejects_oversized_and_bad_sizes_before_any_launch():
    lib = _lib.load()
    big = _params(L=300000, H=16, topk=8)
    assert lib.s3r_workspace_bytes(ctypes.byref(big)) > _lib.S3R_STATIC_WORKSPACE_BYTES
    assert lib.s3r_sparse_attn_fwd_static(ctypes.byref(big), A16, A16, A16, A16, A16, None,
                                          None) == _lib.S3R_ERR_WORKSPACE
    bad = _params(d=128)
    assert lib.s3r_sparse_attn_fwd_static(ctypes.byref(bad), A16, A16, A16, A16, A16, None,
                                          None) == _lib.S3R_ERR_UNSUPPORTED


def test_static_entry_point_needs_a_status_word_and_rejects_save_for_backward():
    lib = _lib.load()
    # no status word: the array's own word is invisible to the caller, so a timeout would be lost
    assert lib.s3r_sparse_attn_fwd_static(ctypes.byref(_params()), A16, A16, A16, A16, A16, None,
                                          None) == _lib.S3R_ERR_INVALID_ARG
    # what a saving forward keeps would live in the shared array, out of the backward's reach
    save = _params(flags=_lib.S3R_FLAG_SAVE_FOR_BWD, dev_status=A16.value)
    assert lib.s3r_sparse_attn_fwd_static(ctypes.byref(save), A16, A16, A16, A16, A16, None,
                                          None) == _lib.S3R_ERR_UNSUPPORTED


def test_last_device_error_rejects_bad_flag_words():
    lib = _lib.load()
    assert lib.s3r_last_device_error(None, None) == _lib.S3R_ERR_INVALID_ARG
    assert lib.s3r_last_device_error(ctypes.c_void_p((1 << 20) + 2), None) == _lib.S3R_ERR_INVALID_ARG


def test_num_key_blocks_of_the_geometries():
    lib = _lib.load()
    # 1-D: ceil(L / b)
    assert lib.s3r_num_key_blocks(ctypes.byref(_params(L=1000, block=64))) == 16
    # VGGT layout: 4 views of 5 special tokens + 37 x 37 patches, 8 x 8 windows: 1 + 5 * 5 a view
    vggt = _params(L=4 * 1374, block=64, grid_h=37, grid_w=37, special=5, win_h=8)
    assert lib.s3r_num_key_blocks(ctypes.byref(vggt)) == 4 * 26
    # no special tokens, 4 x 8 windows on 10 x 13: 3 x 2 windows a view
    assert lib.s3r_num_key_blocks(ctypes.byref(
        _params(L=2 * 130, block=32, grid_h=10, grid_w=13, special=0, win_h=4))) == 2 * 6
    assert lib.s3r_num_key_blocks(ctypes.byref(_params(L=0))) == 0
    cfg = api.Config(L=4 * 1374, H=16, block=64, topk=16, grid_h=37, grid_w=37, special=5, win_h=8)
    assert cfg.nb == 104


def test_sel_attn_rejects_windows_narrower_than_8_before_any_launch():
    lib = _lib.load()
    narrow = _params(L=2 * 130, block=32, topk=2, grid_h=10, grid_w=13, special=0, win_h=8)  # 8 x 4
    assert lib.s3r_sel_attn(ctypes.byref(narrow), A16, A16, A16, A16, A16, None) == _lib.S3R_ERR_UNSUPPORTED
