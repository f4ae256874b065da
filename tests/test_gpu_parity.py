"""GPU parity: every entry point of libs3r.so against the fp64 CPU oracle, element by element, on
seeded synthetic inputs (ragged tails, degenerate sizes, dense selection, tie-heavy scores,
planted well-separated selections). Each call goes through the C ABI via the ctypes binding.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_global_attention_s3r_b200 import _lib, api, synth

from parity import (GAP_EXACT, bf16_ulp, check_close, check_output, check_pooled,
                    check_selection, f64)

pytestmark = pytest.mark.gpu

CASES = {  # name: (L, H, b, k, seed)
    "tiny": (1024, 2, 64, 4, 0),
    "ragged_b64": (1000, 2, 64, 5, 1),
    "ragged_b32_odd_k": (1000, 2, 32, 7, 2),
    "ragged_b128": (1300, 3, 128, 3, 3),
    "single_partial_block": (17, 1, 64, 1, 4),
    "one_token": (1, 2, 32, 1, 5),
    "tail_of_one_row": (65, 1, 32, 3, 6),
    "dense_selection": (1000, 2, 64, 16, 7),  # k = nb
    "multi_tile_keys": (9000, 2, 32, 9, 8),  # nb = 282: several 64-key tiles + ragged tile
    "k_above_32": (3000, 2, 32, 40, 9),  # the fused path materialises the scores for k > 32
}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda")


def inputs(name, device):
    L, H, b, k, seed = CASES[name]
    x = synth.make_inputs(L, H, 64, b, seed)
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    pb = O.Problem(L, H, 64, b, k)
    d = {n: getattr(x, n).to(device) for n in ("q", "k", "v", "gates")}
    return cfg, pb, x, d


@pytest.mark.parametrize("name", list(CASES))
def test_compress_kv(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    kc, vc = api.compress_kv(cfg, d["k"], d["v"])
    torch.cuda.synchronize()
    for got, src in ((kc, x.k), (vc, x.v)):
        ref = O.pool(pb, O.bf16_bits(src))
        exact = check_pooled(f64(got), ref)
        assert exact >= 0.999 or got.numel() < 20000 and exact >= 0.99, exact


@pytest.mark.parametrize("name", list(CASES))
def test_cmp_attn_and_score(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    kc, vc = api.compress_kv(cfg, d["k"], d["v"])
    o, lse, scores = api.cmp_attn_and_score(cfg, d["q"], kc, vc)
    torch.cuda.synchronize()
    rlse, ro, rs = O.cmp_attn(pb, O.bf16_bits(x.q), f64(kc), f64(vc))  # same pooled operands
    check_close("lse", f64(lse), rlse, 2e-5)
    rowmax = rs.max(-1, keepdims=True)
    err = np.abs(f64(scores) - rs)
    assert np.all(err <= 1e-5 * rowmax + 1e-9), float((err / (rowmax + 1e-30)).max())
    check_close("o_cmp", f64(o), ro, 2.0 ** -8 * np.abs(f64(vc)).max() + 1e-6, rl2=4e-3)


@pytest.mark.parametrize("name", list(CASES))
def test_topk_blocks_bit_exact(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    kc, vc = O.pool(pb, O.bf16_bits(x.k)), O.pool(pb, O.bf16_bits(x.v))
    _, _, rs = O.cmp_attn(pb, O.bf16_bits(x.q), kc, vc)
    s32 = rs.astype(np.float32)
    for scores in (s32, np.round(s32 * 4) / 4):  # the second is full of exact ties
        scores = np.ascontiguousarray(scores, np.float32)
        got = api.topk_blocks(cfg, torch.from_numpy(scores).to(dev)).cpu().numpy()
        want, _ = O.topk(scores.astype(np.float64), cfg.topk)  # the same fp32 values
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("k,forced", [(1, 0), (32, 0), (33, 0), (40, 5), (64, 0), (65, 2),
                                     (128, 0), (129, 0), (256, 0), (257, 3)])
def test_topk_adversarial_orders_bit_exact(dev, k, forced):
    """Score rows built against the streaming top-k: ascending scores (every element beats the
    running k-th key, so the candidate buffer overflows and is merged again and again),
    descending, all equal (the lowest indices win), a few distinct values repeated, and random.
    The k values take each size of the warp kernel's sorted list (32, 64, 128, 256) at and past
    its bounds; k = 257 takes the block-wide radix-select kernel. Rows of 3001 scores start at
    every 4-byte offset of a 16-byte line, so the unaligned head and tail are exercised.
    Bit-exact against the oracle's top-k on the same fp32 values."""
    g = torch.Generator().manual_seed(100 + k)
    nb = 3001
    cfg = api.Config(L=nb * 32, H=1, block=32, topk=k, forced=forced)
    rows = torch.stack([
        torch.linspace(0.0, 1.0, nb),
        torch.linspace(1.0, 0.0, nb),
        torch.full((nb,), 0.25),
        torch.randint(0, 4, (nb,), generator=g).float() / 4,
        torch.rand(nb, generator=g),
    ])
    full = torch.zeros((1, cfg.nqb, nb))
    full[0, :rows.shape[0]] = rows
    got = api.topk_blocks(cfg, full.to(dev))[0, :rows.shape[0]].cpu().numpy()
    want, _ = O.topk(rows.double().numpy(), k, forced)
    np.testing.assert_array_equal(got, want)


def test_topk_large_k_unsorted_and_max_blocks(dev):
    g = torch.Generator().manual_seed(9)
    # k > 2048: the set is exact, emitted in ascending index order
    L, b, k = 3000 * 64, 64, 2500
    cfg = api.Config(L=L, H=1, block=b, topk=k)
    s = torch.rand((1, cfg.nqb, cfg.nb), generator=g)
    s[0, :5] = torch.round(s[0, :5] * 3) / 3  # heavy ties in a few rows
    got = api.topk_blocks(cfg, s.to(dev)).cpu().numpy()
    want, _ = O.topk(s.double().numpy(), k)
    np.testing.assert_array_equal(got, np.sort(want, -1))
    # the largest nb this build accepts (shared-memory staging at its limit)
    nb = _lib.S3R_MAX_BLOCKS
    cfg = api.Config(L=nb * 32, H=1, block=32, topk=32)
    rows = torch.rand((1, 4, nb), generator=g)
    full = torch.zeros((1, cfg.nqb, nb))
    full[:, :4] = rows
    got = api.topk_blocks(cfg, full.to(dev))[:, :4].cpu().numpy()
    want, _ = O.topk(rows.double().numpy(), 32)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("name", list(CASES))
def test_sel_attn(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    rng = np.random.default_rng(CASES[name][-1])
    idx = np.stack([np.stack([rng.permutation(cfg.nb)[:cfg.topk] for _ in range(cfg.nqb)])
                    for _ in range(cfg.H)]).astype(np.int32)
    idx[:, -1, 0] = cfg.nb - 1 if cfg.nb - 1 not in idx[:, -1] else idx[:, -1, 0]
    o = api.sel_attn(cfg, d["q"], d["k"], d["v"], torch.from_numpy(idx).to(dev))
    torch.cuda.synchronize()
    ref = O.sel_attn(pb, O.bf16_bits(x.q), O.bf16_bits(x.k), O.bf16_bits(x.v), idx)
    check_close("o_sel", f64(o), ref, 2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6, rl2=4e-3)


def test_sel_attn_debug_checks_flag_bad_indices(dev):
    """An out-of-range index is skipped (its block contributes nothing) and, with debug checks,
    reported in the device status word; reading the word clears it."""
    cfg0, pb, x, d = inputs("ragged_b64", dev)
    k = cfg0.topk
    cfg = api.Config(L=cfg0.L, H=cfg0.H, block=cfg0.block, topk=k, debug_checks=True)
    idx = np.tile(np.arange(k, dtype=np.int32), (cfg.H, cfg.nqb, 1))
    idx[0, 3, 1] = cfg.nb + 7
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    o = api.sel_attn(cfg, d["q"], d["k"], d["v"], torch.from_numpy(idx).to(dev), dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_BAD_INDEX
    assert api.read_device_status(word) == 0
    keep = [c for c in range(k) if c != 1]  # head 0, block 3 without the bad entry
    ref = O.sel_attn(O.Problem(cfg.L, cfg.H, 64, cfg.block, k - 1), O.bf16_bits(x.q),
                     O.bf16_bits(x.k), O.bf16_bits(x.v),
                     np.ascontiguousarray(idx[:, 3:4, keep]), qblocks=[3])
    check_close("o_sel(bad block skipped)", f64(o)[3 * 64:4 * 64, 0], ref[:, 0],
                2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6)


@pytest.mark.parametrize("name", ["tiny", "ragged_b32_odd_k", "ragged_b128"])
def test_gate_combine(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    g = torch.Generator().manual_seed(1)
    oc = torch.randn((cfg.L, cfg.H, 64), generator=g) * 0.01
    os_ = torch.randn((cfg.L, cfg.H, 64), generator=g) * 0.01
    gates = x.gates.clone()
    gates[:5] = 0.0
    gates[5:10, :, 0], gates[5:10, :, 1] = -60.0, 60.0
    out = api.gate_combine(cfg, oc.to(dev), os_.to(dev), gates.to(dev))
    ref = O.combine(oc.double().numpy(), os_.double().numpy(), gates.numpy())
    got = f64(out)
    assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + 1e-7)


def _fused(cfg, d):
    idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=d["q"].device)
    out = api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=idx)
    torch.cuda.synchronize()
    return f64(out), idx.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_sparse_attn_fwd_whole_path(dev, name):
    cfg, pb, x, d = inputs(name, dev)
    out, idx = _fused(cfg, d)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy())
    stats = check_selection(idx, ref.idx, ref.gap, ref.scores, cfg.topk)
    cond = O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx, pooled=(ref.kc, ref.vc))
    check_output(out, cond.out)
    if stats["sets_equal"] == 1.0:
        check_output(out, ref.out)


def test_planted_selection_is_exact(dev):
    L, H, b, k = 4096, 2, 64, 4
    x = synth.make_planted(L, H, 64, b, seed=100)
    cfg, pb = api.Config(L=L, H=H, block=b, topk=k), O.Problem(L, H, 64, b, k)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    out, idx = _fused(cfg, d)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy())
    stats = check_selection(idx, ref.idx, ref.gap, ref.scores, k)
    assert stats["gap_separated"] >= 0.9, stats
    check_output(out, O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx).out)


def test_uniform_keys_select_the_lowest_indices(dev):
    """All keys equal: every block score ties exactly, so the tie rule alone decides: 0..k-1."""
    L, H, b, k = 1000, 2, 64, 5
    x = synth.make_inputs(L, H, 64, b, seed=11)
    kappa = x.k[0:1]
    kk = kappa.expand(L, H, 64).contiguous()
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    d = {"q": x.q.to(dev), "k": kk.to(dev), "v": x.v.to(dev), "gates": x.gates.to(dev)}
    out, idx = _fused(cfg, d)
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(k), idx.shape))
    pb = O.Problem(L, H, 64, b, k)
    ref = O.sparse_attn(pb, *[O.bf16_bits(t) for t in (x.q, kk, x.v)], x.gates.numpy())
    check_output(out, ref.out)


def test_dense_selection_equals_dense_attention(dev):
    """k = nb: the selection branch is ordinary attention over all L tokens (torch SDPA fp64)."""
    L, H, b = 777, 2, 32
    x = synth.make_inputs(L, H, 64, b, seed=12)
    cfg = api.Config(L=L, H=H, block=b, topk=-(-L // b))
    idx = torch.arange(cfg.nb, dtype=torch.int32).expand(H, cfg.nqb, cfg.nb).contiguous()
    o = api.sel_attn(cfg, x.q.to(dev), x.k.to(dev), x.v.to(dev), idx.to(dev))
    q, k, v = (t.double().permute(1, 0, 2)[None] for t in (x.q, x.k, x.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[0].permute(1, 0, 2).numpy()
    check_close("dense", f64(o), ref, 2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6, rl2=4e-3)


@pytest.mark.parametrize("name,launches", [("tiny", 3), ("k_above_32", 4)])
def test_launch_counter_counts_kernels(dev, name, launches):
    cfg, pb, x, d = inputs(name, dev)
    n0 = _lib.kernel_launches()
    api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"])
    torch.cuda.synchronize()
    assert _lib.kernel_launches() - n0 == launches


@pytest.mark.parametrize("name", ["tiny", "ragged_b32_odd_k", "multi_tile_keys", "dense_selection"])
def test_streaming_topk_equals_the_topk_kernel(dev, name):
    """The top-k the compressed kernel keeps on the fly equals s3r_topk_blocks on the same
    (bit-identical) scores, order included."""
    cfg, pb, x, d = inputs(name, dev)
    kc, vc = api.compress_kv(cfg, d["k"], d["v"])
    _, _, scores = api.cmp_attn_and_score(cfg, d["q"], kc, vc)
    want = api.topk_blocks(cfg, scores)
    got = torch.empty_like(want)
    api.sparse_attn_fwd(cfg, d["q"], d["k"], d["v"], d["gates"], idx_out=got)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy(), want.cpu().numpy())


def test_bounded_wait_timeout_is_reported_and_the_context_survives(dev):
    """A wait that nothing satisfies expires after its limit: the kernel records
    S3R_DEV_TIMEOUT in the status word, unwinds and frees its TMEM; the next call works."""
    cfg0, pb, x, d = inputs("ragged_b64", dev)
    kc, vc = api.compress_kv(cfg0, d["k"], d["v"])
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    bad = api.Config(L=cfg0.L, H=cfg0.H, block=cfg0.block, topk=cfg0.topk, test_timeout=True)
    api.cmp_attn_and_score(bad, d["q"], kc, vc, dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_TIMEOUT
    o, lse, scores = api.cmp_attn_and_score(cfg0, d["q"], kc, vc, dev_status=word)
    assert api.read_device_status(word) == 0
    rlse, ro, rs = O.cmp_attn(pb, O.bf16_bits(x.q), f64(kc), f64(vc))
    check_close("lse after a timeout", f64(lse), rlse, 2e-5)


def test_selection_bounded_wait_timeout_is_reported_and_the_context_survives(dev):
    """The selection kernel's softmax warps wait on a barrier nothing signals: the MMA issuer and
    the gather producer give up on their own bounded waits, drain what they issued, the kernel
    records S3R_DEV_TIMEOUT and frees its TMEM; the next call is correct."""
    cfg0, pb, x, d = inputs("ragged_b32_odd_k", dev)
    rng = np.random.default_rng(3)
    idx = np.stack([np.stack([rng.permutation(cfg0.nb)[:cfg0.topk] for _ in range(cfg0.nqb)])
                    for _ in range(cfg0.H)]).astype(np.int32)
    idx_d = torch.from_numpy(idx).to(dev)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    bad = api.Config(L=cfg0.L, H=cfg0.H, block=cfg0.block, topk=cfg0.topk, test_timeout=True)
    api.sel_attn(bad, d["q"], d["k"], d["v"], idx_d, dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_TIMEOUT
    o = api.sel_attn(cfg0, d["q"], d["k"], d["v"], idx_d, dev_status=word)
    assert api.read_device_status(word) == 0
    ref = O.sel_attn(pb, O.bf16_bits(x.q), O.bf16_bits(x.k), O.bf16_bits(x.v), idx)
    check_close("o_sel after a timeout", f64(o), ref, 2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6,
                rl2=4e-3)


# --------------------------------------------------------------------------------------------
# VGGT variant: the reference frame's blocks open every selection list
# --------------------------------------------------------------------------------------------

FORCED = {  # name: (L, H, b, k, forced, seed)
    "vggt_4_views": (4 * 1374, 2, 64, 16, 22, 20),  # P = 1374 tokens per view, F = ceil(P/b)
    "forced_b32_odd_list": (2000, 2, 32, 5, 6, 21),  # F + k odd: the last step is half empty
    "forced_k_above_32": (3000, 2, 32, 36, 5, 22),  # top-k kernel on the materialised scores
    "forced_plus_k_is_nb": (1000, 2, 64, 12, 4, 23),  # F + k = nb: dense selection
}


def forced_inputs(name, device):
    L, H, b, k, F, seed = FORCED[name]
    x = synth.make_inputs(L, H, 64, b, seed)
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=F)
    pb = O.Problem(L, H, 64, b, k, forced=F)
    d = {n: getattr(x, n).to(device) for n in ("q", "k", "v", "gates")}
    return cfg, pb, x, d


@pytest.mark.parametrize("name", list(FORCED))
def test_forced_whole_path(dev, name):
    cfg, pb, x, d = forced_inputs(name, dev)
    out, idx = _fused(cfg, d)
    assert idx.shape == (cfg.H, cfg.nqb, cfg.forced + cfg.topk)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy())
    stats = check_selection(idx, ref.idx, ref.gap, ref.scores, cfg.topk, cfg.forced)
    cond = O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx, pooled=(ref.kc, ref.vc))
    check_output(out, cond.out)
    if stats["sets_equal"] == 1.0:
        check_output(out, ref.out)


@pytest.mark.parametrize("name", list(FORCED))
def test_forced_topk_blocks_bit_exact(dev, name):
    cfg, pb, x, d = forced_inputs(name, dev)
    kc, vc = O.pool(pb, O.bf16_bits(x.k)), O.pool(pb, O.bf16_bits(x.v))
    _, _, rs = O.cmp_attn(pb, O.bf16_bits(x.q), kc, vc)
    s32 = rs.astype(np.float32)
    for scores in (s32, np.round(s32 * 4) / 4):
        scores = np.ascontiguousarray(scores, np.float32)
        got = api.topk_blocks(cfg, torch.from_numpy(scores).to(dev)).cpu().numpy()
        want, _ = O.topk(scores.astype(np.float64), cfg.topk, cfg.forced)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("name", ["vggt_4_views", "forced_b32_odd_list"])
def test_forced_sel_attn(dev, name):
    cfg, pb, x, d = forced_inputs(name, dev)
    rng = np.random.default_rng(FORCED[name][-1])
    F, k = cfg.forced, cfg.topk
    idx = np.stack([np.stack([np.concatenate([np.arange(F), F + rng.permutation(cfg.nb - F)[:k]])
                              for _ in range(cfg.nqb)]) for _ in range(cfg.H)]).astype(np.int32)
    o = api.sel_attn(cfg, d["q"], d["k"], d["v"], torch.from_numpy(idx).to(dev))
    torch.cuda.synchronize()
    ref = O.sel_attn(pb, O.bf16_bits(x.q), O.bf16_bits(x.k), O.bf16_bits(x.v), idx)
    check_close("o_sel", f64(o), ref, 2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6, rl2=4e-3)


# --------------------------------------------------------------------------------------------
# 2-D windows on each view's patch grid (special tokens as a block of their own)
# --------------------------------------------------------------------------------------------

WINDOWS = {  # name: (views, special, grid_h, grid_w, b, win_h, H, k, forced_views, seed)
    "vggt_4_views_8x8": (4, 5, 37, 37, 64, 8, 2, 16, 0, 30),
    "vggt_ref_view_forced": (4, 5, 37, 37, 64, 8, 2, 12, 1, 31),
    "odd_grid_4x8_b32": (3, 3, 10, 13, 32, 4, 2, 5, 0, 32),
    "wide_8x16_b128": (2, 0, 20, 35, 128, 8, 2, 3, 0, 33),
    "k_above_32_4x8": (6, 5, 16, 16, 32, 4, 2, 40, 0, 34),
    "one_view_grid_smaller_than_window": (1, 2, 3, 5, 64, 8, 2, 1, 0, 36),
    "special_fills_a_block": (3, 32, 6, 9, 32, 4, 2, 4, 0, 37),
    "forced_views_k_above_32": (5, 5, 16, 16, 32, 4, 2, 36, 1, 38),
}


def window_inputs(name, device):
    N, special, gh, gw, b, wh, H, k, fv, seed = WINDOWS[name]
    L = N * (special + gh * gw)
    geo = dict(grid_h=gh, grid_w=gw, special=special, win_h=wh)
    per_view = api.Config(L=L, H=H, block=b, topk=1, **geo).nb // N
    F = fv * per_view
    x = synth.make_inputs(L, H, 64, b, seed)
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=F, **geo)
    pb = O.Problem(L, H, 64, b, k, forced=F, **geo)
    assert cfg.nb == pb.nb
    d = {n: getattr(x, n).to(device) for n in ("q", "k", "v", "gates")}
    return cfg, pb, x, d


@pytest.mark.parametrize("name", list(WINDOWS))
def test_windows_compress_kv(dev, name):
    cfg, pb, x, d = window_inputs(name, dev)
    kc, vc = api.compress_kv(cfg, d["k"], d["v"])
    torch.cuda.synchronize()
    for got, src in ((kc, x.k), (vc, x.v)):
        exact = check_pooled(f64(got), O.pool(pb, O.bf16_bits(src)))
        assert exact >= 0.99, exact


@pytest.mark.parametrize("name", list(WINDOWS))
def test_windows_sel_attn_gathers_from_k_and_v(dev, name):
    """The step entry point gathers window rows straight from K, V [L, H, 64]."""
    cfg, pb, x, d = window_inputs(name, dev)
    rng = np.random.default_rng(WINDOWS[name][-1])
    n = cfg.nsel
    idx = np.stack([np.stack([rng.permutation(cfg.nb)[:n] for _ in range(cfg.nqb)])
                    for _ in range(cfg.H)]).astype(np.int32)
    o = api.sel_attn(cfg, d["q"], d["k"], d["v"], torch.from_numpy(idx).to(dev))
    torch.cuda.synchronize()
    ref = O.sel_attn(pb, O.bf16_bits(x.q), O.bf16_bits(x.k), O.bf16_bits(x.v), idx)
    check_close("o_sel", f64(o), ref, 2.0 ** -8 * np.abs(f64(x.v)).max() + 1e-6, rl2=4e-3)


@pytest.mark.parametrize("name", list(WINDOWS))
def test_windows_whole_path(dev, name):
    cfg, pb, x, d = window_inputs(name, dev)
    out, idx = _fused(cfg, d)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy())
    stats = check_selection(idx, ref.idx, ref.gap, ref.scores, cfg.topk, cfg.forced)
    cond = O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx, pooled=(ref.kc, ref.vc))
    check_output(out, cond.out)
    if stats["sets_equal"] == 1.0:
        check_output(out, ref.out)


def test_windows_one_patch_high_match_1d_blocks_bit_for_bit(dev):
    """Windows 1 x b on a grid b-multiple wide without special tokens are the 1-D blocks: the
    fused path must produce identical bits either way."""
    N, gh, gw, b, k, H = 3, 5, 128, 64, 6, 2
    L = N * gh * gw
    x = synth.make_inputs(L, H, 64, b, 35)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    one = api.Config(L=L, H=H, block=b, topk=k)
    two = api.Config(L=L, H=H, block=b, topk=k, grid_h=gh, grid_w=gw, special=0, win_h=1)
    assert one.nb == two.nb
    o1, i1 = _fused(one, d)
    o2, i2 = _fused(two, d)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_array_equal(o1, o2)


def test_host_pipeline_matches_device_calls(dev):
    """Steps submitted from pinned host memory through the overlapped pipeline give the same
    outputs as device-resident calls, step by step, with every slot reused at least once."""
    L, H, b, k = 3000, 2, 64, 5
    cfg = api.Config(L=L, H=H, block=b, topk=k)
    steps = [synth.make_inputs(L, H, 64, b, 40 + s) for s in range(5)]
    want = []
    sa = api.SparseAttention(cfg, dev)
    for x in steps:
        want.append(sa(*(getattr(x, n).to(dev) for n in ("q", "k", "v", "gates"))).cpu())
    pipe = api.HostPipeline(cfg, dev)
    host_out = [torch.empty((L, H, 64), dtype=torch.bfloat16).pin_memory() for _ in steps]
    host_in = [[getattr(x, n).pin_memory() for n in ("q", "k", "v", "gates")] for x in steps]
    for ins, o in zip(host_in, host_out):
        pipe.submit(*ins, o)
    pipe.synchronize()
    for got, ref in zip(host_out, want):
        assert torch.equal(got, ref)


# --------------------------------------------------------------------------------------------
# the single fused kernel: compressed branch, streamed top-k and selection in one CTA
# --------------------------------------------------------------------------------------------

SINGLE = ["tiny", "ragged_b64", "ragged_b32_odd_k", "ragged_b128", "single_partial_block",
          "one_token", "tail_of_one_row", "dense_selection", "multi_tile_keys"]


def _single(cfg):
    return api.Config(**{**cfg.__dict__, "single_kernel": True})


@pytest.mark.parametrize("name", SINGLE)
def test_single_kernel_whole_path(dev, name):
    """Two launches (pooling, then one kernel per query tile): the same lists as the three-launch
    path (the compressed branch is the same arithmetic), and the output against the oracle."""
    cfg, pb, x, d = inputs(name, dev)
    n0 = _lib.kernel_launches()
    out, idx = _fused(_single(cfg), d)
    assert _lib.kernel_launches() - n0 == 2
    out3, idx3 = _fused(cfg, d)
    np.testing.assert_array_equal(idx, idx3)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx)
    check_output(out, ref.out)
    # O_cmp is kept as bf16 on chip: within a bf16 rounding of the three-launch output
    assert np.abs(out - out3).max() <= 2.0 ** -7 * np.abs(out3).max() + 1e-6


@pytest.mark.parametrize("name", ["vggt_4_views", "forced_b32_odd_list", "forced_plus_k_is_nb"])
def test_single_kernel_forced(dev, name):
    cfg, pb, x, d = forced_inputs(name, dev)
    out, idx = _fused(_single(cfg), d)
    out3, idx3 = _fused(cfg, d)
    np.testing.assert_array_equal(idx, idx3)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    check_output(out, O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx).out)


@pytest.mark.parametrize("name", ["vggt_4_views_8x8", "vggt_ref_view_forced", "odd_grid_4x8_b32",
                                  "wide_8x16_b128", "special_fills_a_block"])
def test_single_kernel_windows(dev, name):
    cfg, pb, x, d = window_inputs(name, dev)
    out, idx = _fused(_single(cfg), d)
    out3, idx3 = _fused(cfg, d)
    np.testing.assert_array_equal(idx, idx3)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    check_output(out, O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx).out)


def test_single_kernel_timeout_is_reported_and_the_context_survives(dev):
    cfg, pb, x, d = inputs("ragged_b64", dev)
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    bad = api.Config(**{**cfg.__dict__, "single_kernel": True, "test_timeout": True})
    api.sparse_attn_fwd(bad, d["q"], d["k"], d["v"], d["gates"], dev_status=word)
    assert api.read_device_status(word) & _lib.S3R_DEV_TIMEOUT
    out, idx = _fused(_single(cfg), d)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    check_output(out, O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx).out)


# --------------------------------------------------------------------------------------------
# seeded random configurations across every option at once
# --------------------------------------------------------------------------------------------

def _random_config(seed):
    """A small configuration drawn from every axis: block size, top-k on both sides of 32,
    forced blocks, 1-D or 2-D geometry (special tokens, cut windows), single kernel or not."""
    rng = np.random.default_rng(1000 + seed)
    b = int(rng.choice([32, 64, 128]))
    H = int(rng.integers(1, 4))
    geo = {}
    if rng.random() < 0.5:
        wh = int(rng.choice([w for w in (1, 2, 4, 8) if b // w >= 8]))
        gh, gw = int(rng.integers(1, 24)), int(rng.integers(1, 40))
        special = int(rng.integers(0, min(b, 6) + 1))
        views = int(rng.integers(1, 5))
        geo = dict(grid_h=gh, grid_w=gw, special=special, win_h=wh)
        L = views * (special + gh * gw)
    else:
        L = int(rng.integers(1, 5000))
    nb = api.Config(L=L, H=H, block=b, topk=1, **geo).nb
    forced = int(rng.integers(0, min(nb - 1, 8) + 1)) if nb > 1 and rng.random() < 0.4 else 0
    k = int(rng.integers(1, min(nb - forced, 40) + 1))
    single = bool(k <= 32 and rng.random() < 0.5)
    return dict(L=L, H=H, block=b, topk=k, forced=forced, single_kernel=single, **geo)


@pytest.mark.parametrize("seed", range(16))
def test_random_configurations(dev, seed):
    kw = _random_config(seed)
    cfg = api.Config(**kw)
    x = synth.make_inputs(cfg.L, cfg.H, 64, cfg.block, 2000 + seed)
    d = {n: getattr(x, n).to(dev) for n in ("q", "k", "v", "gates")}
    out, idx = _fused(cfg, d)
    pk = {k: v for k, v in kw.items() if k not in ("block", "topk", "single_kernel", "L", "H")}
    pb = O.Problem(cfg.L, cfg.H, 64, cfg.block, cfg.topk, **pk)
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    ref = O.sparse_attn(pb, *bits, x.gates.numpy())
    check_selection(idx, ref.idx, ref.gap, ref.scores, cfg.topk, cfg.forced)
    cond = O.sparse_attn(pb, *bits, x.gates.numpy(), idx_given=idx, pooled=(ref.kc, ref.vc))
    check_output(out, cond.out)
