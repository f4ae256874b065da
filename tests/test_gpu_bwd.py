"""GPU parity of the backward (s3r_sparse_attn_bwd) against the fp64 oracle's gradients.

The selection lists are the forward call's own (idx_out), handed to both sides; the oracle gets
the pooled K/V rounded to bf16 as the forward used them (its gradient passes that rounding
straight through, like the library's).

Tolerance (bf16 operands, fp32 accumulation): the kernels round g*P and dS to bf16 before the
tensor-core products (relative error 2^-9 per element) and take D = g <dout, O> from the fp32
forward outputs, whose own error is about 2^-8 of |V| (bf16 P in the forward products). Both
enter every gradient at about 2^-8 relative, so each of dq, dk, dv, dgates must satisfy
rel-L2 <= 1e-2 and max-abs <= 2e-2 * max|reference| + 1e-6 (a wrong index, sign or dropped term
gives errors of order 1). The absolute 1e-6 covers gradients that are exactly zero: with a single
key a branch's P is 1 and dS = P (g dP' - D) vanishes, but in fp32 the difference g dP' - D keeps
a rounding residue of about 2^-24 |dP| (measured: 4.5e-9 in dq at L = 1).
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_global_attention_s3r_b200 import api, synth

from parity import check_grad, f64

pytestmark = pytest.mark.gpu


CASES = {  # name: (L, H, b, k, forced, seed)
    "ragged_b64": (1000, 2, 64, 5, 0, 41),
    "ragged_b32_odd_k": (1000, 2, 32, 7, 0, 42),
    "ragged_b128": (1300, 3, 128, 3, 0, 43),
    "multi_tile_keys": (9000, 2, 32, 9, 0, 44),   # nb = 282: several key tiles of both kernels
    "dense_selection": (1000, 2, 64, 16, 0, 45),  # k = nb
    "single_partial_block": (17, 1, 64, 1, 0, 46),
    "one_token": (1, 2, 32, 1, 0, 47),
    "tail_of_one_row": (65, 1, 32, 3, 0, 48),
    "forced_b32": (2000, 2, 32, 5, 6, 49),        # reference-frame blocks in every list
    "vggt_4_views": (4 * 1374, 2, 64, 16, 22, 50),
    # 8 summary tiles of one head: the dKc/dVc kernel splits its walk over the queries into the
    # most pieces it takes, 16, added back in order
    "sixteen_pieces": (40000, 1, 64, 8, 0, 58),
}

WINDOWS = {  # name: (views, special, grid_h, grid_w, b, win_h, H, k, forced_views, seed)
    "vggt_8x8_ref_view": (4, 5, 37, 37, 64, 8, 2, 12, 1, 51),
    "odd_grid_4x8_b32": (3, 3, 10, 13, 32, 4, 2, 5, 0, 52),
    "wide_8x16_b128": (2, 0, 20, 35, 128, 8, 2, 3, 0, 53),
    "narrow_8x4_b32": (2, 2, 10, 13, 32, 8, 2, 3, 0, 54),  # windows narrower than 8 patches
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda")


def _dout(L, H, seed):
    g = torch.Generator().manual_seed(1000 + seed)
    return torch.randn((L, H, 64), generator=g).to(torch.bfloat16)


_check = check_grad


def _run(dev, cfg, pb, x, seed):
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=idx)
    dout = _dout(cfg.L, cfg.H, seed)
    dq, dk, dv, dg = api.sparse_attn_bwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx,
                                         dout.to(dev))
    torch.cuda.synchronize()
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.backward(pb, *bits, x.gates.numpy(), idx.cpu().numpy(), dout.double().numpy())
    for n, got, want in (("dq", dq, ref.dq), ("dk", dk, ref.dk), ("dv", dv, ref.dv),
                         ("dgates", dg, ref.dgates)):
        _check(n, got, want)


@pytest.mark.parametrize("name", list(CASES))
def test_bwd_matches_oracle(dev, name):
    L, H, b, k, F, seed = CASES[name]
    x = synth.make_inputs(L, H, 64, b, seed)
    _run(dev, api.Config(L=L, H=H, block=b, topk=k, forced=F),
         O.Problem(L, H, 64, b, k, forced=F), x, seed)


@pytest.mark.parametrize("name", list(WINDOWS))
def test_bwd_windows_match_oracle(dev, name):
    N, special, gh, gw, b, wh, H, k, fv, seed = WINDOWS[name]
    L = N * (special + gh * gw)
    geo = dict(grid_h=gh, grid_w=gw, special=special, win_h=wh)
    F = fv * (api.Config(L=L, H=H, block=b, topk=1, **geo).nb // N)
    x = synth.make_inputs(L, H, 64, b, seed)
    _run(dev, api.Config(L=L, H=H, block=b, topk=k, forced=F, **geo),
         O.Problem(L, H, 64, b, k, forced=F, **geo), x, seed)


def test_bwd_unselected_blocks_get_only_the_pooled_gradient(dev):
    """Selection lists naming only block 0: every other key block's tokens receive exactly their
    share of the compressed branch's dKc / n_j (the selection branch adds nothing there)."""
    L, H, b, k = 640, 1, 64, 1
    x = synth.make_inputs(L, H, 64, b, 55)
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    pb = O.Problem(L, H, 64, b, k)
    idx = torch.zeros((H, cfg.nqb, 1), dtype=torch.int32)
    dout = _dout(L, H, 55)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    dq, dk, dv, dg = api.sparse_attn_bwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx.to(dev),
                                         dout.to(dev))
    torch.cuda.synchronize()
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.backward(pb, *bits, x.gates.numpy(), idx.numpy(), dout.double().numpy())
    for n, got, want in (("dq", dq, ref.dq), ("dk", dk, ref.dk), ("dv", dv, ref.dv)):
        _check(n, got, want)
    # tokens of blocks 1.. get the pooled gradient only: equal within each block
    g = f64(dk)[b:].reshape(L // b - 1, b, H, 64)
    assert np.abs(g - g[:, :1]).max() <= 1e-6 * max(1.0, np.abs(g).max())


def test_bwd_autograd_function(dev):
    """SparseAttentionFunction: forward = the fused path, backward = s3r_sparse_attn_bwd."""
    L, H, b, k = 1000, 2, 64, 4
    x = synth.make_inputs(L, H, 64, b, 56)
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    leaves = [getattr(x, n).to(dev).requires_grad_() for n in ("q", "k", "v", "gates")]
    out = api.SparseAttentionFunction.apply(*leaves, cfg)
    dout = _dout(L, H, 56).to(dev)
    out.backward(dout)
    idx = torch.empty((H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    ref_out = api.sparse_attn_fwd(cfg, *[t.detach() for t in leaves], idx_out=idx)
    assert torch.equal(out.detach(), ref_out)
    dq, dk, dv, dg = api.sparse_attn_bwd(cfg, *[t.detach() for t in leaves], idx, dout)
    # two backward calls may add query blocks into a key block in different orders (atomic
    # fill), so the bf16 casts may differ by one rounding step
    for leaf, want in zip(leaves, (dq, dk, dv, dg)):
        assert leaf.grad.dtype == leaf.dtype
        torch.testing.assert_close(leaf.grad.float(), want.float(), rtol=8e-3, atol=1e-6)


@pytest.mark.parametrize("name", ["ragged_b32_odd_k", "forced_b32", "vggt_4_views"])
def test_bwd_from_saved_forward(dev, name):
    """save_for_backward: the forward's output is unchanged, and the backward on its saved
    tensors (no recompute) matches the oracle and the recomputing backward."""
    import dataclasses

    L, H, b, k, F, seed = CASES[name]
    x = synth.make_inputs(L, H, 64, b, seed)
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=F)
    save = dataclasses.replace(cfg, save_for_backward=True)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    idx = torch.empty((H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    out = api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=idx)
    ws = torch.empty(api.bwd_workspace_bytes(save), dtype=torch.uint8, device=dev)
    idx_s = torch.empty_like(idx)
    out_s = api.sparse_attn_fwd(save, d["q"], d["k"], d["v"], d["gates"], workspace=ws,
                                idx_out=idx_s)
    assert torch.equal(out_s, out) and torch.equal(idx_s, idx)
    dout = _dout(L, H, seed).to(dev)
    saved = api.sparse_attn_bwd(save, d["q"], d["k"], d["v"], d["gates"], idx_s, dout,
                                workspace=ws)
    again = api.sparse_attn_bwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx, dout)
    torch.cuda.synchronize()
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.backward(O.Problem(L, H, 64, b, k, forced=F), *bits, x.gates.numpy(),
                     idx.cpu().numpy(), dout.cpu().double().numpy())
    for n, got, other, want in zip(("dq", "dk", "dv", "dgates"), saved, again,
                                   (ref.dq, ref.dk, ref.dv, ref.dgates)):
        _check(n, got, want)
        # the same kernels on the same values; only the order of additions into a key block's
        # dk, dv may differ (atomic fill)
        torch.testing.assert_close(got, other, rtol=1e-5, atol=1e-6)


def test_bwd_debug_checks_flag_bad_indices(dev):
    """A list entry outside [0, nb) is skipped by the backward and, with debug checks, raises
    S3R_DEV_BAD_INDEX in the caller's status word; without them the word stays clear."""
    import dataclasses

    from sparse_global_attention_s3r_b200 import _lib

    L, H, b, k, F, seed = CASES["ragged_b64"]
    x = synth.make_inputs(L, H, 64, b, seed)
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    idx = torch.empty((H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=idx)
    idx[0, 3, 1] = cfg.nb + 7
    dout = _dout(L, H, seed).to(dev)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    api.sparse_attn_bwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx, dout, dev_status=word)
    assert api.read_device_status(word) == 0
    checked = dataclasses.replace(cfg, debug_checks=True)
    grads = api.sparse_attn_bwd(checked, d["q"], d["k"], d["v"], d["gates"], idx, dout,
                                dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_BAD_INDEX
    for g in grads:
        assert torch.isfinite(g).all()


def test_bwd_status_word_stays_clear(dev):
    L, H, b, k = 1000, 2, 64, 4
    x = synth.make_inputs(L, H, 64, b, 57)
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    idx = torch.empty((H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=idx)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    api.sparse_attn_bwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx,
                        _dout(L, H, 57).to(dev), dev_status=word)
    assert api.read_device_status(word) == 0


def test_bwd_bounded_wait_timeout_is_reported_and_the_context_survives(dev):
    """S3R_FLAG_TEST_TIMEOUT makes the backward's tensor-core kernels (dq, dKc/dVc, dk/dv) wait
    on a barrier nothing signals, with a 1 ms limit. After a saving forward the backward runs only
    those kernels, so the status word must carry S3R_DEV_TIMEOUT from them; the next backward on
    the same workspace must then be correct again."""
    import dataclasses

    from sparse_global_attention_s3r_b200 import _lib

    L, H, b, k, F, seed = CASES["ragged_b32_odd_k"]
    x = synth.make_inputs(L, H, 64, b, seed)
    save = api.Config(L=L, H=H, block=b, topk=k, forced=F, save_for_backward=True)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    ws = torch.empty(api.bwd_workspace_bytes(save), dtype=torch.uint8, device=dev)
    idx = torch.empty((H, save.nqb, save.nsel), dtype=torch.int32, device=dev)
    api.sparse_attn_fwd(save, d["q"], d["k"], d["v"], d["gates"], workspace=ws, idx_out=idx)
    dout = _dout(L, H, seed).to(dev)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    timed_out = dataclasses.replace(save, test_timeout=True)
    api.sparse_attn_bwd(timed_out, d["q"], d["k"], d["v"], d["gates"], idx, dout, workspace=ws,
                        dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_TIMEOUT
    grads = api.sparse_attn_bwd(save, d["q"], d["k"], d["v"], d["gates"], idx, dout,
                                workspace=ws, dev_status=word)
    assert api.read_device_status(word) == 0
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.backward(O.Problem(L, H, 64, b, k, forced=F), *bits, x.gates.numpy(),
                     idx.cpu().numpy(), dout.cpu().double().numpy())
    for n, got, want in zip(("dq", "dk", "dv", "dgates"), grads,
                            (ref.dq, ref.dk, ref.dv, ref.dgates)):
        _check(n, got, want)
