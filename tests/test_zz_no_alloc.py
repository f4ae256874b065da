"""s3r_sparse_attn_fwd_static: the whole path for callers that cannot allocate device memory.

Such callers (a host framework that owns all device memory and hands plugins no workspace, or a
loop that must not allocate once running) call this entry point, which takes its scratch memory
from an array built into the library instead of a workspace argument. This file is collected last
on purpose, so that a run stopping at its first failure has already run every other test.

Each call goes through the C ABI; its output must equal the allocating entry point's output on
the same inputs, within the tolerances of the other parity tests, on two calls in a row with
different inputs (the shared array keeps the previous call's contents).
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_global_attention_s3r_b200 import _lib, api, synth

from parity import check_output

pytestmark = pytest.mark.gpu


def _call_static(cfg, x, dev):
    out = torch.empty((cfg.L, cfg.H, 64), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((cfg.H, cfg.nqb, cfg.topk), dtype=torch.int32, device=dev)
    p = cfg.params()
    st = _lib.load().s3r_sparse_attn_fwd_static(
        ctypes.byref(p), ctypes.c_void_p(x["q"].data_ptr()), ctypes.c_void_p(x["k"].data_ptr()),
        ctypes.c_void_p(x["v"].data_ptr()), ctypes.c_void_p(x["gates"].data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.S3R_OK, _lib.status_string(st)
    return out, idx


def _call_allocating(cfg, x, dev):
    idx = torch.empty((cfg.H, cfg.nqb, cfg.topk), dtype=torch.int32, device=dev)
    out = api.sparse_attn_fwd(cfg, x["q"], x["k"], x["v"], x["gates"], idx_out=idx)
    return out, idx


def test_static_workspace_entry_point_matches_the_allocating_one():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    cases = [(1000, 2, 64, 5, 21), (3000, 4, 32, 7, 22)]  # ragged tails, different sizes
    for L, H, b, k, seed in cases:  # two calls in a row on the shared array
        cfg = api.Config(L=L, H=H, block=b, topk=k)
        assert api.workspace_bytes(cfg) <= _lib.S3R_STATIC_WORKSPACE_BYTES
        g = synth.make_inputs(L, H, 64, b, seed)
        x = {n: getattr(g, n).to(dev) for n in ("q", "k", "v", "gates")}
        out_s, idx_s = _call_static(cfg, x, dev)
        out_a, idx_a = _call_allocating(cfg, x, dev)
        torch.cuda.synchronize()
        check_output(out_s.double().cpu().numpy(), out_a.double().cpu().numpy())
        np.testing.assert_array_equal(idx_s.cpu().numpy(), idx_a.cpu().numpy())


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
