"""s3r_sparse_attn_fwd_static: the whole path for callers that cannot allocate device memory.

Such callers (a host framework that owns all device memory and hands plugins no workspace, or a
loop that must not allocate once running) call this entry point, which takes its scratch memory
from an array built into the library instead of a workspace argument. This file is collected last
on purpose, so that a run stopping at its first failure has already run every other test.

Each call goes through the C ABI. Both entry points run the same kernels on the same inputs, so
the output and the selection lists must be identical, bit for bit, on several calls in a row with
different sizes and paths (the shared array keeps the previous call's contents). A bounded wait
that expires must reach the caller's status word.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_global_attention_s3r_b200 import _lib, api, synth

pytestmark = pytest.mark.gpu


def _call_static(cfg, x, dev, word):
    out = torch.empty((cfg.L, cfg.H, 64), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    p = cfg.params(word)
    st = _lib.load().s3r_sparse_attn_fwd_static(
        ctypes.byref(p), ctypes.c_void_p(x["q"].data_ptr()), ctypes.c_void_p(x["k"].data_ptr()),
        ctypes.c_void_p(x["v"].data_ptr()), ctypes.c_void_p(x["gates"].data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.S3R_OK, _lib.status_string(st)
    return out, idx


def _call_allocating(cfg, x, dev):
    idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    out = api.sparse_attn_fwd(cfg, x["q"], x["k"], x["v"], x["gates"], idx_out=idx)
    return out, idx


def _inputs(cfg, seed, dev):
    g = synth.make_inputs(cfg.L, cfg.H, 64, cfg.block, seed)
    return {n: getattr(g, n).to(dev) for n in ("q", "k", "v", "gates")}


def test_static_workspace_entry_point_matches_the_allocating_one():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    cases = [  # ragged tails, different sizes and paths, each right after the previous call
        api.Config(L=1000, H=2, block=64, topk=5),
        api.Config(L=3000, H=4, block=32, topk=7),
        api.Config(L=700, H=2, block=64, topk=3, single_kernel=True),   # after a larger call
        api.Config(L=4 * 300, H=2, block=64, topk=4, forced=5),         # forced blocks
        api.Config(L=1500, H=3, block=32, topk=40),                     # k > 32: score matrix
    ]
    for n, cfg in enumerate(cases):
        assert api.workspace_bytes(cfg) <= _lib.S3R_STATIC_WORKSPACE_BYTES
        x = _inputs(cfg, 21 + n, dev)
        out_s, idx_s = _call_static(cfg, x, dev, word)
        out_a, idx_a = _call_allocating(cfg, x, dev)
        torch.cuda.synchronize()
        assert api.read_device_status(word) == 0
        np.testing.assert_array_equal(idx_s.cpu().numpy(), idx_a.cpu().numpy())
        assert torch.equal(out_s.view(torch.int16), out_a.view(torch.int16)), f"case {n}"


def test_static_workspace_entry_point_reports_a_timeout_in_the_callers_word():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    cfg = api.Config(L=1000, H=2, block=64, topk=5)
    x = _inputs(cfg, 31, dev)
    _call_static(api.Config(L=1000, H=2, block=64, topk=5, test_timeout=True), x, dev, word)
    torch.cuda.synchronize()
    assert api.read_device_status(word) & _lib.S3R_DEV_TIMEOUT
    # the context survives and the next call is correct
    out_s, idx_s = _call_static(cfg, x, dev, word)
    out_a, idx_a = _call_allocating(cfg, x, dev)
    torch.cuda.synchronize()
    assert api.read_device_status(word) == 0
    np.testing.assert_array_equal(idx_s.cpu().numpy(), idx_a.cpu().numpy())
    assert torch.equal(out_s.view(torch.int16), out_a.view(torch.int16))


def test_static_workspace_entry_point_rejects_sizes_beyond_its_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = api.Config(L=300000, H=16, block=64, topk=8)
    assert api.workspace_bytes(cfg) > _lib.S3R_STATIC_WORKSPACE_BYTES
    p = cfg.params()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call is rejected first
    st = _lib.load().s3r_sparse_attn_fwd_static(ctypes.byref(p), fake, fake, fake, fake, fake,
                                                None, None)
    assert st == _lib.S3R_ERR_WORKSPACE
