"""Pins of the fp64 CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against a closed form, an invariant, brute force over every
candidate, or a library routine (torch SDPA / topk / bf16 cast, all on CPU in fp64), chosen so that
a plausible slip in the oracle (a dropped term, a wrong index, a swapped operand, a tail divided by
the wrong count) fails at least one of them. tests/test_oracle_mutants.py plants such slips and
checks that they are caught.

Method: gist.science summary of "Speed3R: Sparse Feed-forward 3D Reconstruction Models",
"Technische samenvatting" -> "Methodologie" §1 (compression branch: average pooling and a score
matrix; selection branch: fine attention on the top-k) and §2 (gated aggregation).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


# --------------------------------------------------------------------------------------------
# helpers (value <-> bf16 bits; none of them implements a step of the method)
# --------------------------------------------------------------------------------------------

def bits_of(x) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable in bf16 (asserted)."""
    a = torch.as_tensor(np.asarray(x, dtype=np.float32))
    b = a.to(torch.bfloat16)
    assert torch.equal(b.float(), a), "test value not representable in bf16"
    return O.bf16_bits(b)


def values_of(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def rand_bits(shape, seed, scale=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if scale is not None:
        x = x * scale
    return O.bf16_bits(x.to(torch.bfloat16))


def sdpa64(q, k, v, scale, mask=None):
    """torch SDPA in fp64 on [L, H, d] arrays -> [L, H, dv]."""
    tq = torch.from_numpy(np.ascontiguousarray(q)).double().permute(1, 0, 2)[None]
    tk = torch.from_numpy(np.ascontiguousarray(k)).double().permute(1, 0, 2)[None]
    tv = torch.from_numpy(np.ascontiguousarray(v)).double().permute(1, 0, 2)[None]
    m = None if mask is None else torch.from_numpy(mask)
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


# --------------------------------------------------------------------------------------------
# bf16 rounding
# --------------------------------------------------------------------------------------------

def test_round_bf16_matches_library_cast_on_floats():
    g = torch.Generator().manual_seed(11)
    x = torch.randn(4000, generator=g) * torch.exp2(torch.randint(-40, 40, (4000,), generator=g))
    # constructed halfway and near-halfway float32 patterns
    hi = torch.randint(0, 1 << 15, (3000,), generator=g, dtype=torch.int64) << 16
    lows = torch.tensor([0x8000, 0x7FFF, 0x8001, 0x0000, 0xFFFF], dtype=torch.int64)
    pats = (hi[:, None] | lows[None, :]).reshape(-1)
    pats = pats[(pats >> 23) & 0xFF != 0xFF]  # finite only
    y = pats.to(torch.int32).view(torch.float32)
    allx = torch.cat([x, y])
    want = allx.to(torch.bfloat16).double().numpy()
    got = np.array([O.round_bf16(float(v)) for v in allx.tolist()])
    np.testing.assert_array_equal(got, want)


def test_round_bf16_rounds_the_exact_double_once():
    # just above / below the halfway point between 1 and 1 + 2^-7: a float32 round trip would
    # land exactly on the tie and round to even (1.0) in both cases
    assert O.round_bf16(1 + 2**-8 + 2**-40) == 1 + 2**-7
    assert O.round_bf16(1 + 2**-8 - 2**-40) == 1.0
    assert O.round_bf16(1 + 2**-8) == 1.0  # tie -> even
    assert O.round_bf16(1 + 3 * 2**-8) == 1 + 2**-6  # tie -> even
    assert O.round_bf16(-(1 + 3 * 2**-8)) == -(1 + 2**-6)
    # subnormal range: quantum 2^-133
    assert O.round_bf16(2.0**-134) == 0.0
    assert O.round_bf16(3 * 2.0**-134) == 2.0**-132
    assert O.round_bf16(5 * 2.0**-135) == 2.0**-133


# --------------------------------------------------------------------------------------------
# pooling (compression branch, average pooling)
# --------------------------------------------------------------------------------------------

@pytest.mark.parametrize("L,b", [(200, 64), (256, 64), (97, 32), (300, 128), (1, 64)])
def test_pool_constant_blocks(L, b):
    H, d = 2, 8
    nb = -(-L // b)
    rng = np.random.default_rng(L + b)
    const = rng.integers(-64, 64, size=(nb, H, d)) / 8.0  # bf16-exact
    x = np.repeat(const, b, axis=0)[:L]
    pb = O.Problem(L, H, d, b, 1)
    for exact in (True, False):
        np.testing.assert_array_equal(O.pool(pb, bits_of(x), exact=exact), const)


@pytest.mark.parametrize("L,b", [(200, 64), (97, 32), (300, 128), (129, 128)])
def test_pool_linear_ramp_gives_midpoint_of_valid_tokens(L, b):
    H, d = 3, 4
    t = np.arange(L)
    # value = position inside the block + 10*e + 100*h: integers, exact in bf16 up to 256
    x = (t % b)[:, None, None] + 10.0 * np.arange(d)[None, None, :] + 0.0 * np.arange(H)[None, :, None]
    x = x + 40.0 * np.arange(H)[None, :, None]
    pb = O.Problem(L, H, d, b, 1)
    got = O.pool(pb, bits_of(x), exact=True)
    nb = -(-L // b)
    for j in range(nb):
        n = min(b, L - j * b)
        want = (n - 1) / 2.0 + 10.0 * np.arange(d)[None, :] + 40.0 * np.arange(H)[:, None]
        np.testing.assert_array_equal(got[j], want)
    # rounded mode: the exact mean rounded once to bf16 (a library cast of the exact float32 value)
    got_r = O.pool(pb, bits_of(x), exact=False)
    want_r = torch.from_numpy(got.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got_r, want_r)


def test_pool_rounded_is_within_half_ulp_of_exact():
    L, H, d, b = 333, 2, 16, 64
    x = rand_bits((L, H, d), 5, scale=0.125)
    pb = O.Problem(L, H, d, b, 1)
    ex = O.pool(pb, x, exact=True)
    rd = O.pool(pb, x, exact=False)
    # bf16 representable
    np.testing.assert_array_equal(
        torch.from_numpy(rd).float().to(torch.bfloat16).double().numpy(), rd)
    ulp = np.exp2(np.floor(np.log2(np.abs(ex) + 1e-300)) - 7)
    assert np.all(np.abs(rd - ex) <= 0.5 * ulp * (1 + 1e-12))


# --------------------------------------------------------------------------------------------
# compression branch: attention to block summaries and the score matrix
# --------------------------------------------------------------------------------------------

def _setup(L, H, d, b, k, seed, qscale=None):
    pb = O.Problem(L, H, d, b, k)
    s = 1 / math.sqrt(d) if qscale is None else qscale
    q = rand_bits((L, H, d), seed, s)
    kk = rand_bits((L, H, d), seed + 1, 1 / math.sqrt(d))
    v = rand_bits((L, H, d), seed + 2, 1 / math.sqrt(d))
    return pb, q, kk, v


@pytest.mark.parametrize("L,b,k", [(1000, 64, 4), (1024, 64, 4), (500, 32, 3)])
def test_cmp_uniform_keys_closed_form(L, b, k):
    """All keys equal: every summary equals that key, so p = 1/nb, lse = s + log nb,
    o_cmp = mean of the pooled V, scores tie at rows/nb and the top-k is 0..k-1."""
    H, d = 2, 16
    pb = O.Problem(L, H, d, b, k)
    kappa = values_of(rand_bits((H, d), 3, 0.5))
    kk = bits_of(np.broadcast_to(kappa, (L, H, d)))
    q = rand_bits((L, H, d), 4, 0.5)
    v = rand_bits((L, H, d), 5, 0.5)
    kc = O.pool(pb, kk)
    vc = O.pool(pb, v)
    lse, o_cmp, scores = O.cmp_attn(pb, q, kc, vc)
    qv = values_of(q)
    s = pb.softmax_scale * np.einsum("lhd,hd->hl", qv, kappa)
    np.testing.assert_allclose(lse, s + math.log(pb.nb), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_cmp, np.broadcast_to(vc.mean(axis=0), o_cmp.shape), atol=1e-14)
    rows = np.array([min(64, L - 64 * i) for i in range(pb.nqb)], np.float64)
    np.testing.assert_allclose(scores, np.broadcast_to((rows / pb.nb)[None, :, None], scores.shape),
                               rtol=1e-13)
    idx, gap = O.topk(scores, k)
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(k), idx.shape))


def test_cmp_two_level_keys_closed_form():
    """Summaries are kappa on a set A of blocks and 0 elsewhere: p_A = e^s / (|A| e^s + nb - |A|)."""
    L, H, d, b, k = 700, 2, 8, 64, 3
    pb = O.Problem(L, H, d, b, k)
    nb = pb.nb
    A = [1, 4, 5, 10]  # includes the ragged last block (10)
    kappa = values_of(rand_bits((H, d), 7, 1.0))
    x = np.zeros((L, H, d))
    for j in A:
        x[j * b:(j + 1) * b] = kappa
    q = rand_bits((L, H, d), 8, 0.7)
    v = rand_bits((L, H, d), 9, 0.5)
    kc = O.pool(pb, bits_of(x))
    vc = O.pool(pb, v)
    lse, o_cmp, scores = O.cmp_attn(pb, q, kc, vc)
    s = pb.softmax_scale * np.einsum("lhd,hd->hl", values_of(q), kappa)  # [H, L]
    Z = len(A) * np.exp(s) + (nb - len(A))
    pA, p0 = np.exp(s) / Z, 1.0 / Z
    np.testing.assert_allclose(lse, np.log(Z), atol=1e-12)
    inA = np.zeros(nb, bool)
    inA[A] = True
    want_o = (pA.T[:, :, None] * vc[inA].sum(0)[None] + p0.T[:, :, None] * vc[~inA].sum(0)[None])
    np.testing.assert_allclose(o_cmp, want_o, atol=1e-14)
    want_s = np.zeros((H, pb.nqb, nb))
    for i in range(pb.nqb):
        r = slice(64 * i, min(L, 64 * i + 64))
        want_s[:, i, :] = np.where(inA[None, :], pA[:, r].sum(1)[:, None], p0[:, r].sum(1)[:, None])
    np.testing.assert_allclose(scores, want_s, rtol=1e-13)


def test_cmp_scores_sum_to_rows_of_each_query_block():
    L, H, d, b = 1000, 2, 64, 64
    pb, q, kk, v = _setup(L, H, d, b, 4, 21)
    _, _, scores = O.cmp_attn(pb, q, O.pool(pb, kk), O.pool(pb, v))
    rows = np.array([min(64, L - 64 * i) for i in range(pb.nqb)], np.float64)
    np.testing.assert_allclose(scores.sum(-1), np.broadcast_to(rows, (H, pb.nqb)), rtol=1e-13)


@pytest.mark.parametrize("L,b", [(1000, 64), (777, 32), (900, 128)])
def test_cmp_matches_library_attention_fp64(L, b):
    """o_cmp = SDPA(q, K~, V~); SDPA(q, K~, I) returns the probability matrix itself, whose
    query-block sums are the scores and whose first column fixes lse = s_q0 - log p_q0."""
    H, d = 2, 64
    pb, q, kk, v = _setup(L, H, d, b, 4, 31, qscale=1.0)  # larger logits than the workload
    kc, vc = O.pool(pb, kk), O.pool(pb, v)
    lse, o_cmp, scores = O.cmp_attn(pb, q, kc, vc)
    qv = values_of(q)
    np.testing.assert_allclose(o_cmp, sdpa64(qv, kc, vc, pb.softmax_scale), rtol=0, atol=1e-13)
    eye = np.broadcast_to(np.eye(pb.nb)[:, None, :], (pb.nb, H, pb.nb))
    P = sdpa64(qv, kc, eye, pb.softmax_scale)  # [L, H, nb]
    for i in range(pb.nqb):
        np.testing.assert_allclose(scores[:, i, :], P[64 * i:64 * i + 64].sum(0), rtol=1e-11,
                                   atol=1e-15)
    s0 = pb.softmax_scale * np.einsum("lhd,hd->hl", qv, kc[0])
    np.testing.assert_allclose(lse, s0 - np.log(P[:, :, 0].T), atol=1e-11)


def test_cmp_sampled_blocks_equal_full_run():
    L, H, d, b = 1000, 2, 32, 64
    pb, q, kk, v = _setup(L, H, d, b, 4, 41)
    kc, vc = O.pool(pb, kk), O.pool(pb, v)
    lse, o, sc = O.cmp_attn(pb, q, kc, vc)
    pick = [15, 3, 0]  # includes the ragged last query block
    lse2, o2, sc2 = O.cmp_attn(pb, q, kc, vc, qblocks=pick)
    rows = pb.rows_of(pick)
    np.testing.assert_array_equal(lse2, lse[:, rows])
    np.testing.assert_array_equal(o2, o[rows])
    np.testing.assert_array_equal(sc2, sc[:, pick])


# --------------------------------------------------------------------------------------------
# per-query-block top-k
# --------------------------------------------------------------------------------------------

def test_topk_equals_best_subset_by_brute_force():
    """The top-k set maximises the score sum over all k-subsets; among equal sums the
    lexicographically smallest index tuple (= lower index first on ties). Integer-valued scores
    make every sum exact and ties frequent."""
    rng = np.random.default_rng(0)
    n = 9
    for trial in range(60):
        row = rng.integers(0, 4, size=n).astype(np.float64)
        for k in range(1, n + 1):
            best = max(itertools.combinations(range(n), k),
                       key=lambda c: (sum(row[list(c)]), tuple(-x for x in c)))
            idx, gap = O.topk(row[None], k)
            assert sorted(idx[0].tolist()) == list(best), (row, k)
            # order: descending score, ties by lower index
            order = sorted(best, key=lambda j: (-row[j], j))
            assert idx[0].tolist() == order
            srt = np.sort(row)[::-1]
            want_gap = math.inf if k == n else srt[k - 1] - srt[k]
            assert gap[0] == want_gap


def test_topk_matches_library_topk_without_ties():
    g = torch.Generator().manual_seed(3)
    s = torch.rand(40, 300, generator=g, dtype=torch.float64)
    for k in (1, 7, 32, 300):
        idx, _ = O.topk(s.numpy(), k)
        want = torch.topk(s, k, dim=-1, sorted=True).indices.numpy()
        np.testing.assert_array_equal(idx, want)


def test_topk_with_forced_blocks_by_brute_force():
    """VGGT variant (reference-frame blocks always kept): the lists open with blocks 0..F-1 in
    order, and the remaining k entries are the best k-subset of blocks F..n-1 by brute force,
    ordered by descending score, ties by lower index; the gap is taken among those blocks."""
    rng = np.random.default_rng(5)
    n = 9
    for trial in range(40):
        row = rng.integers(0, 4, size=n).astype(np.float64)
        for forced in range(0, 4):
            for k in range(1, n - forced + 1):
                rest = range(forced, n)
                best = max(itertools.combinations(rest, k),
                           key=lambda c: (sum(row[list(c)]), tuple(-x for x in c)))
                idx, gap = O.topk(row[None], k, forced)
                assert idx.shape == (1, forced + k)
                assert idx[0, :forced].tolist() == list(range(forced))
                assert idx[0, forced:].tolist() == sorted(best, key=lambda j: (-row[j], j))
                srt = np.sort(row[forced:])[::-1]
                assert gap[0] == (math.inf if k == n - forced else srt[k - 1] - srt[k])


def test_topk_forced_blocks_scores_have_no_effect():
    """Raising or lowering the forced blocks' own scores changes no list: they are kept without
    competing, and they never take one of the k places."""
    g = torch.Generator().manual_seed(9)
    s = torch.rand(30, 50, generator=g, dtype=torch.float64).numpy()
    for forced, k in ((1, 5), (7, 12), (20, 30)):
        base, gap = O.topk(s, k, forced)
        for fill in (1e9, -1e9, 0.0):
            t = s.copy()
            t[:, :forced] = fill
            idx, gap2 = O.topk(t, k, forced)
            np.testing.assert_array_equal(idx, base)
            np.testing.assert_array_equal(gap2, gap)
        # forced = 0 is the plain top-k
    np.testing.assert_array_equal(O.topk(s, 5, 0)[0], O.topk(s, 5)[0])


# --------------------------------------------------------------------------------------------
# selection branch
# --------------------------------------------------------------------------------------------

@pytest.mark.parametrize("L,b", [(1000, 64), (777, 32), (900, 128)])
def test_sel_with_every_block_equals_dense_library_attention(L, b):
    H, d = 2, 64
    pb0, q, kk, v = _setup(L, H, d, b, 1, 51, qscale=1.0)
    pb = O.Problem(L, H, d, b, pb0.nb)
    idx = np.broadcast_to(np.arange(pb.nb, dtype=np.int32), (H, pb.nqb, pb.nb))
    o = O.sel_attn(pb, q, kk, v, idx)
    want = sdpa64(values_of(q), values_of(kk), values_of(v), pb.softmax_scale)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("L,b,k", [(1000, 64, 4), (777, 32, 5), (900, 128, 2)])
def test_sel_matches_library_attention_under_block_mask(L, b, k):
    """Arbitrary distinct selections, the ragged last block included: SDPA with a boolean mask
    that admits exactly the tokens of the selected blocks of each query's block."""
    H, d = 2, 64
    pb, q, kk, v = _setup(L, H, d, b, k, 61, qscale=1.0)
    rng = np.random.default_rng(k)
    idx = np.stack([np.stack([rng.permutation(pb.nb)[:k] for _ in range(pb.nqb)])
                    for _ in range(H)]).astype(np.int32)
    idx[:, -1, 0] = pb.nb - 1 if (pb.nb - 1) not in idx[:, -1, 1:] else idx[:, -1, 0]
    o = O.sel_attn(pb, q, kk, v, idx)
    qv, kv, vv = values_of(q), values_of(kk), values_of(v)
    for h in range(H):
        mask = np.zeros((L, L), bool)
        for i in range(pb.nqb):
            for j in idx[h, i]:
                mask[64 * i:64 * i + 64, j * b:min(L, j * b + b)] = True
        want = sdpa64(qv[:, h:h + 1], kv[:, h:h + 1], vv[:, h:h + 1], pb.softmax_scale, mask[None, None])
        np.testing.assert_allclose(o[:, h:h + 1], want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("L,b,forced", [(1000, 64, 3), (777, 32, 10), (900, 128, 1)])
def test_sel_forced_plus_topk_covering_every_block_equals_dense_attention(L, b, forced):
    """With F forced blocks and k = nb - F the lists cover every block: the selection branch is
    dense attention (library SDPA in fp64), whatever order the top-k part has."""
    H, d = 2, 64
    pb0, q, kk, v = _setup(L, H, d, b, 1, 53, qscale=1.0)
    nb = pb0.nb
    pb = O.Problem(L, H, d, b, nb - forced, forced=forced)
    rng = np.random.default_rng(forced)
    lists = [np.concatenate([np.arange(forced), forced + rng.permutation(nb - forced)])
             for _ in range(H * pb.nqb)]
    idx = np.stack(lists).reshape(H, pb.nqb, nb).astype(np.int32)
    o = O.sel_attn(pb, q, kk, v, idx)
    want = sdpa64(values_of(q), values_of(kk), values_of(v), pb.softmax_scale)
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-13)


def test_pipeline_with_forced_blocks_attends_to_the_reference_frame():
    """Whole path of the VGGT variant on 4 views of 160 tokens, b = 32: the reference frame
    (view 0, blocks 0..4) opens every list; the selection output equals masked library attention
    over the forced tokens plus the blocks of the oracle's own top-k; the compression branch and
    the scores are those of the plain path."""
    P, N, H, d, b, k = 160, 4, 2, 64, 32, 3
    L = P * N
    forced = -(-P // b)
    pb, q, kk, v = _setup(L, H, d, b, k, 57, qscale=0.8)
    pbf = O.Problem(L, H, d, b, k, forced=forced)
    gates = _gates(L, H, 58)
    plain = O.sparse_attn(pb, q, kk, v, gates)
    res = O.sparse_attn(pbf, q, kk, v, gates)
    np.testing.assert_array_equal(res.scores, plain.scores)
    np.testing.assert_array_equal(res.o_cmp, plain.o_cmp)
    assert res.idx.shape == (H, pbf.nqb, forced + k)
    assert (res.idx[..., :forced] == np.arange(forced)).all()
    assert (res.idx[..., forced:] >= forced).all()
    qv, kv, vv = values_of(q), values_of(kk), values_of(v)
    for h in range(H):
        mask = np.zeros((L, L), bool)
        for i in range(pbf.nqb):
            for j in res.idx[h, i]:
                mask[64 * i:64 * i + 64, j * b:min(L, j * b + b)] = True
        assert mask[:, :P].all()
        want = sdpa64(qv[:, h:h + 1], kv[:, h:h + 1], vv[:, h:h + 1], pbf.softmax_scale,
                      mask[None, None])
        np.testing.assert_allclose(res.o_sel[:, h:h + 1], want, rtol=0, atol=1e-13)


def test_sel_block_order_and_duplicates_do_not_matter():
    L, H, d, b, k = 640, 1, 32, 64, 3
    pb, q, kk, v = _setup(L, H, d, b, k, 71)
    idx = np.array([[[2, 5, 7]] * pb.nqb], np.int32)
    a = O.sel_attn(pb, q, kk, v, idx)
    b_ = O.sel_attn(pb, q, kk, v, idx[:, :, ::-1].copy())
    np.testing.assert_allclose(a, b_, atol=1e-15)
    dup = np.array([[[2, 5, 5]] * pb.nqb], np.int32)
    two = O.Problem(L, H, d, b, 2)
    c = O.sel_attn(pb, q, kk, v, dup)
    e = O.sel_attn(two, q, kk, v, np.array([[[2, 5]] * pb.nqb], np.int32))
    np.testing.assert_allclose(c, e, atol=1e-15)


# --------------------------------------------------------------------------------------------
# gated aggregation
# --------------------------------------------------------------------------------------------

def test_combine_gate_limits_and_midpoint():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((50, 3, 8))
    b = rng.standard_normal((50, 3, 8))
    z = np.zeros((50, 3, 2), np.float32)
    np.testing.assert_allclose(O.combine(a, b, z), 0.5 * (a + b), rtol=1e-15)
    lim = np.zeros_like(z)
    lim[..., 0], lim[..., 1] = -60, 60
    np.testing.assert_allclose(O.combine(a, b, lim), b, rtol=1e-15, atol=1e-25)
    lim[..., 0], lim[..., 1] = 60, -60
    np.testing.assert_allclose(O.combine(a, b, lim), a, rtol=1e-15, atol=1e-25)
    # the two gates are independent: both open -> the plain sum
    lim[..., 0], lim[..., 1] = 60, 60
    np.testing.assert_allclose(O.combine(a, b, lim), a + b, rtol=1e-15)


# --------------------------------------------------------------------------------------------
# the worked example (tests/golden/worked_example.json)
# --------------------------------------------------------------------------------------------

def test_worked_example():
    with open(os.path.join(HERE, "golden", "worked_example.json")) as f:
        ex = json.load(f)
    p = ex["problem"]
    pb = O.Problem(p["L"], p["H"], p["d"], p["block"], p["topk"], qblock=p["qblock"], scale=p["scale"])
    inp = ex["inputs"]
    q = bits_of(np.array(inp["q"], np.float64)[:, None, :])
    k = bits_of(np.array(inp["k"], np.float64)[:, None, :])
    v = bits_of(np.array(inp["v"], np.float64)[:, None, :])
    gates = np.array(inp["gates"], np.float32)[:, None, :]
    r = O.sparse_attn(pb, q, k, v, gates)
    e = ex["expected"]
    np.testing.assert_array_equal(r.kc[:, 0], e["pooled_k"])
    np.testing.assert_array_equal(r.vc[:, 0], e["pooled_v"])
    s = np.array(e["logits"], np.float64)
    P = np.exp(s) / np.exp(s).sum(1, keepdims=True)
    np.testing.assert_allclose(r.lse[0], np.log(np.exp(s).sum(1)), atol=1e-15)
    np.testing.assert_allclose(r.o_cmp[:, 0], P @ np.array(e["pooled_v"], np.float64), atol=1e-15)
    want_scores = np.stack([P[0] + P[1], P[2] + P[3], P[4]])
    np.testing.assert_allclose(r.scores[0], want_scores, atol=1e-15)
    np.testing.assert_array_equal(r.idx[0], e["idx"])
    np.testing.assert_allclose(r.o_sel[:, 0], e["o_sel"], atol=1e-15)
    np.testing.assert_allclose(r.out[:, 0], 0.5 * (r.o_cmp[:, 0] + np.array(e["o_sel"])), atol=1e-15)


# --------------------------------------------------------------------------------------------
# invariances of the whole path
# --------------------------------------------------------------------------------------------

def _pipeline(pb, q, k, v, gates):
    return O.sparse_attn(pb, q, k, v, gates)


def _gates(L, H, seed):
    return torch.randn((L, H, 2), generator=torch.Generator().manual_seed(seed)).numpy()


def test_invariance_tokens_permuted_within_key_blocks():
    """Re-ordering tokens inside every key block (K and V together; on the multi-view layout,
    the order of the views' patches inside a block) changes nothing but summation order."""
    L, H, d, b, k = 1000, 2, 64, 64, 4
    pb, q, kk, v = _setup(L, H, d, b, k, 81, qscale=0.6)
    gates = _gates(L, H, 1)
    rng = np.random.default_rng(2)
    perm = np.concatenate([j * b + rng.permutation(min(b, L - j * b)) for j in range(pb.nb)])
    r0 = _pipeline(pb, q, kk, v, gates)
    r1 = _pipeline(pb, q, kk[perm].copy(), v[perm].copy(), gates)
    np.testing.assert_array_equal(r0.kc, r1.kc)
    np.testing.assert_array_equal(r0.vc, r1.vc)
    np.testing.assert_allclose(r0.scores, r1.scores, rtol=1e-13)
    sep = r0.gap > 1e-9
    np.testing.assert_array_equal(np.sort(r0.idx, -1)[sep], np.sort(r1.idx, -1)[sep])
    np.testing.assert_allclose(r0.out, r1.out, atol=1e-13)


def test_invariance_queries_permuted_within_query_blocks():
    L, H, d, b, k = 1000, 2, 64, 64, 4
    pb, q, kk, v = _setup(L, H, d, b, k, 91, qscale=0.6)
    gates = _gates(L, H, 2)
    rng = np.random.default_rng(3)
    perm = np.concatenate([i * 64 + rng.permutation(min(64, L - i * 64)) for i in range(pb.nqb)])
    r0 = _pipeline(pb, q, kk, v, gates)
    r1 = _pipeline(pb, q[perm].copy(), kk, v, gates[perm].copy())
    np.testing.assert_allclose(r1.scores, r0.scores, rtol=1e-13)
    sep = r0.gap > 1e-9
    np.testing.assert_array_equal(np.sort(r0.idx, -1)[sep], np.sort(r1.idx, -1)[sep])
    np.testing.assert_allclose(r1.out, r0.out[perm], atol=1e-13)
    np.testing.assert_allclose(r1.lse, r0.lse[:, perm], atol=1e-13)


def test_invariance_key_blocks_permuted():
    """Moving whole key blocks permutes the score columns and relabels the selection; the
    outputs do not change."""
    L, H, d, b, k = 1024, 2, 64, 64, 4
    pb, q, kk, v = _setup(L, H, d, b, k, 101, qscale=0.6)
    gates = _gates(L, H, 3)
    rng = np.random.default_rng(4)
    pi = rng.permutation(pb.nb)  # new block pi[j] holds old block j
    tok = np.empty(L, np.int64)
    for j in range(pb.nb):
        tok[pi[j] * b:(pi[j] + 1) * b] = np.arange(j * b, (j + 1) * b)
    r0 = _pipeline(pb, q, kk, v, gates)
    r1 = _pipeline(pb, q, kk[tok].copy(), v[tok].copy(), gates)
    np.testing.assert_allclose(r1.scores[:, :, pi], r0.scores, rtol=1e-13)
    sep = r0.gap > 1e-9
    np.testing.assert_array_equal(np.sort(pi[r0.idx], -1)[sep], np.sort(r1.idx, -1)[sep])
    np.testing.assert_allclose(r1.out, r0.out, atol=1e-13)


def test_heads_are_independent():
    L, H, d, b, k = 700, 3, 32, 64, 3
    pb, q, kk, v = _setup(L, H, d, b, k, 111, qscale=0.8)
    gates = _gates(L, H, 4)
    full = _pipeline(pb, q, kk, v, gates)
    one = O.Problem(L, 1, d, b, k)
    for h in range(H):
        r = _pipeline(one, q[:, h:h + 1].copy(), kk[:, h:h + 1].copy(), v[:, h:h + 1].copy(),
                      gates[:, h:h + 1].copy())
        np.testing.assert_array_equal(r.idx[0], full.idx[h])
        np.testing.assert_array_equal(r.out[:, 0], full.out[:, h])


def test_scale_applies_to_both_branches():
    """(q, scale) and (2q, scale/2) give the same logits exactly, hence identical outputs."""
    L, H, d, b, k = 600, 2, 32, 64, 3
    pb, q, kk, v = _setup(L, H, d, b, k, 121, qscale=0.5)
    gates = _gates(L, H, 5)
    q2 = bits_of(2 * values_of(q))
    a = O.sparse_attn(O.Problem(L, H, d, b, k, scale=0.3), q, kk, v, gates)
    c = O.sparse_attn(O.Problem(L, H, d, b, k, scale=0.15), q2, kk, v, gates)
    np.testing.assert_array_equal(a.idx, c.idx)
    np.testing.assert_array_equal(a.out, c.out)
    # and the scale matters: a different scale changes the compressed output
    e = O.sparse_attn(O.Problem(L, H, d, b, k, scale=0.6), q, kk, v, gates)
    assert np.abs(e.o_cmp - a.o_cmp).max() > 1e-6


# --------------------------------------------------------------------------------------------
# 2-D windows on each view's patch grid
# --------------------------------------------------------------------------------------------

def _geo(N, special, gh, gw, b, win_h, H=2, k=3, forced=0):
    P = special + gh * gw
    return O.Problem(N * P, H, 64, b, k, forced=forced, grid_h=gh, grid_w=gw, special=special,
                     win_h=win_h)


def test_2d_blocks_partition_each_view_into_rectangles():
    """Every token lies in exactly one key block; a block never spans two views; the special
    tokens of a view form one block; every other block is a rectangle of at most win_h x win_w
    patches whose sides are cut only by the grid's right and bottom edges."""
    for N, special, gh, gw, b, wh in [(3, 5, 37, 37, 64, 8), (2, 0, 10, 13, 32, 4),
                                      (2, 3, 9, 17, 128, 8), (1, 1, 5, 5, 32, 1)]:
        pb = _geo(N, special, gh, gw, b, wh)
        P, ww = special + gh * gw, b // wh
        seen = np.zeros(pb.L, np.int64)
        for j in range(pb.nb):
            t = pb.block_tokens(j)
            assert 0 < t.size <= b and np.all(np.diff(t) > 0)
            seen[t] += 1
            view = t // P
            assert np.all(view == view[0])
            off = t - view[0] * P
            if off[0] < special:
                np.testing.assert_array_equal(off, np.arange(special))
                continue
            r, c = (off - special) // gw, (off - special) % gw
            rows, cols = np.unique(r), np.unique(c)
            assert rows.size * cols.size == t.size  # a full rectangle of patches
            assert np.all(np.diff(rows) == 1) and np.all(np.diff(cols) == 1)
            assert rows[0] % wh == 0 and cols[0] % ww == 0
            assert rows.size == min(wh, gh - rows[0]) and cols.size == min(ww, gw - cols[0])
        assert np.all(seen == 1)


def test_2d_windows_of_one_patch_row_equal_1d_blocks():
    """Windows one patch high and b wide on a grid b-multiple wide, with no special tokens, are
    exactly the 1-D blocks of b consecutive tokens: the whole path must agree bit for bit."""
    N, gh, gw, b, k = 2, 6, 128, 64, 3
    pb2 = _geo(N, 0, gh, gw, b, 1, k=k)
    pb1 = O.Problem(pb2.L, 2, 64, b, k)
    assert pb2.nb == pb1.nb
    q, kk, v = (rand_bits((pb2.L, 2, 64), s, 0.7) for s in (91, 92, 93))
    g = _gates(pb2.L, 2, 94)
    a, c = O.sparse_attn(pb2, q, kk, v, g), O.sparse_attn(pb1, q, kk, v, g)
    for name in ("kc", "vc", "lse", "o_cmp", "scores", "idx", "o_sel", "out"):
        np.testing.assert_array_equal(getattr(a, name), getattr(c, name), err_msg=name)


def test_2d_pooling_of_a_ramp_is_the_ramp_at_the_window_centre():
    """K = alpha*row + beta*col + e over the patches and a constant over the special tokens: the
    mean over a (possibly cut) window is the ramp at the mean row and mean column of its patches,
    computed here from the window corners alone."""
    N, special, gh, gw, b, wh = 2, 4, 11, 13, 32, 4
    ww = b // wh
    pb = _geo(N, special, gh, gw, b, wh, H=1)
    P = special + gh * gw
    x = np.zeros((pb.L, 1, 64))
    e = (np.arange(64) % 4) / 2.0  # every value below is a multiple of 1/2 under 32: exact in bf16
    for view in range(N):
        x[view * P:view * P + special, 0, :] = 3.0 + e
        for r in range(gh):
            for c in range(gw):
                x[view * P + special + r * gw + c, 0, :] = 2.0 * r + 0.5 * c + e
    got = O.pool(pb, bits_of(x), exact=True)
    per_view = 1 + (-(-gh // wh)) * (-(-gw // ww))
    for j in range(pb.nb):
        m = j % per_view
        if m == 0:
            np.testing.assert_array_equal(got[j, 0], 3.0 + e)
            continue
        wr, wc = divmod(m - 1, -(-gw // ww))
        r0, r1 = wr * wh, min(gh, wr * wh + wh) - 1
        c0, c1 = wc * ww, min(gw, wc * ww + ww) - 1
        want = 2.0 * (r0 + r1) / 2 + 0.5 * (c0 + c1) / 2 + e
        np.testing.assert_allclose(got[j, 0], want, rtol=0, atol=1e-12)


def test_2d_selection_matches_library_attention_under_window_mask():
    """Selection over windows, cut edge windows and special blocks included: SDPA with a boolean
    mask admitting exactly the selected windows' tokens for the rows of each query block."""
    pb = _geo(2, 5, 9, 11, 32, 4, H=2, k=4)
    q, kk, v = (rand_bits((pb.L, 2, 64), s, 1.0 / 8) for s in (95, 96, 97))
    rng = np.random.default_rng(7)
    idx = np.stack([np.stack([rng.permutation(pb.nb)[:pb.topk] for _ in range(pb.nqb)])
                    for _ in range(2)]).astype(np.int32)
    o = O.sel_attn(pb, q, kk, v, idx)
    qv, kv, vv = values_of(q), values_of(kk), values_of(v)
    for h in range(2):
        mask = np.zeros((pb.L, pb.L), bool)
        for i in range(pb.nqb):
            for j in idx[h, i]:
                mask[64 * i:64 * i + 64, pb.block_tokens(int(j))] = True
        want = sdpa64(qv[:, h:h + 1], kv[:, h:h + 1], vv[:, h:h + 1], pb.softmax_scale,
                      mask[None, None])
        np.testing.assert_allclose(o[:, h:h + 1], want, rtol=0, atol=1e-13)


def test_2d_invariance_patches_permuted_within_windows():
    """Re-ordering the patches inside every window (K and V together) changes nothing but the
    summation order of the pooled means."""
    pb = _geo(2, 5, 9, 11, 32, 4, H=2, k=4)
    q, kk, v = (rand_bits((pb.L, 2, 64), s, 0.7) for s in (98, 99, 100))
    g = _gates(pb.L, 2, 101)
    perm = np.arange(pb.L)
    rng = np.random.default_rng(3)
    for j in range(pb.nb):
        t = pb.block_tokens(j)
        perm[t] = rng.permutation(t)
    a = O.sparse_attn(pb, q, kk, v, g)
    b_ = O.sparse_attn(pb, q, kk[perm], v[perm], g)
    np.testing.assert_allclose(a.kc, b_.kc, atol=1e-2 * np.abs(a.kc).max())
    np.testing.assert_allclose(a.scores, b_.scores, rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(a.out, b_.out, rtol=1e-3, atol=1e-5)


def test_2d_reference_view_forced_covers_every_token_of_view_zero():
    """VGGT variant on windows: forcing the first view's blocks (its special block and all its
    windows) puts every token of view 0, and no token of another view, among the forced tokens."""
    N, special, gh, gw, b, wh = 3, 5, 9, 11, 32, 4
    pb0 = _geo(N, special, gh, gw, b, wh)
    per_view = pb0.nb // N
    pb = _geo(N, special, gh, gw, b, wh, k=3, forced=per_view)
    P = special + gh * gw
    q, kk, v = (rand_bits((pb.L, 2, 64), s, 0.7) for s in (102, 103, 104))
    res = O.sparse_attn(pb, q, kk, v, _gates(pb.L, 2, 105))
    toks = np.concatenate([pb.block_tokens(j) for j in range(per_view)])
    np.testing.assert_array_equal(np.sort(toks), np.arange(P))
    assert (res.idx[..., :per_view] == np.arange(per_view)).all()
    assert (res.idx[..., per_view:] >= per_view).all()


# --------------------------------------------------------------------------------------------
# backward: gradients of the whole path with the selection held fixed
# --------------------------------------------------------------------------------------------
# The path is trained end to end (arXiv abstract of Speed3R), so the oracle also gives the
# gradients of dQ, dK, dV and the gate logits for an upstream gradient dout. The top-k has no
# gradient: the lists are fixed; the bf16 rounding of the pooled K/V is passed straight through,
# so the pins hand the backward the exact fp64 means (pool(..., exact=True)).

def _bwd_inputs(pb, seed, gates=None):
    q = rand_bits((pb.L, pb.H, pb.d), seed, 1.0)
    k = rand_bits((pb.L, pb.H, pb.d), seed + 1, 1.0)
    v = rand_bits((pb.L, pb.H, pb.d), seed + 2, 1.0)
    g = _gates(pb.L, pb.H, seed + 3) if gates is None else gates
    dout = torch.randn((pb.L, pb.H, pb.d), generator=torch.Generator().manual_seed(seed + 4),
                       dtype=torch.float64).numpy()
    return q, k, v, np.ascontiguousarray(g, np.float32), dout


def _bwd(pb, q, k, v, g, idx, dout):
    kc = O.pool(pb, k, exact=True)
    vc = O.pool(pb, v, exact=True)
    return O.backward(pb, q, k, v, g, idx, dout, kc=kc, vc=vc), kc, vc


def _torch_path(pb, q, k, v, g, idx):
    """The forward written with torch ops on fp64 leaves (exact pooling, idx fixed): pooled K/V are
    means of each block's tokens, the compressed branch attends to all of them, the selection
    branch to the tokens of the listed blocks, and sigmoid gates mix the two."""
    blocks = [torch.from_numpy(pb.block_tokens(j)) for j in range(pb.nb)]
    kc = torch.stack([k[t].mean(0) for t in blocks])
    vc = torch.stack([v[t].mean(0) for t in blocks])
    out = []
    for h in range(pb.H):
        rows_h = []
        for i in range(pb.nqb):
            r = slice(i * pb.qblock, min((i + 1) * pb.qblock, pb.L))
            qi = q[r, h]
            oc = torch.softmax(pb.softmax_scale * qi @ kc[:, h].T, -1) @ vc[:, h]
            toks = torch.cat([blocks[j] for j in sorted(set(idx[h, i].tolist()))])
            os_ = torch.softmax(pb.softmax_scale * qi @ k[toks, h].T, -1) @ v[toks, h]
            gi = torch.sigmoid(g[r, h])
            rows_h.append(gi[:, :1] * oc + gi[:, 1:] * os_)
        out.append(torch.cat(rows_h))
    return torch.stack(out, 1)


def _leaves(q, k, v, g):
    return [torch.tensor(values_of(q), requires_grad=True),
            torch.tensor(values_of(k), requires_grad=True),
            torch.tensor(values_of(v), requires_grad=True),
            torch.tensor(g.astype(np.float64), requires_grad=True)]


@pytest.mark.parametrize("pb", [
    O.Problem(200, 2, 16, 32, 3),             # 1-D, ragged tail block and query block
    O.Problem(300, 2, 16, 32, 2, forced=2),   # reference-frame blocks always kept
    O.Problem(246, 2, 16, 32, 3, forced=1, grid_h=10, grid_w=12, special=3, win_h=4),  # 2-D
])
def test_bwd_equals_autograd_of_the_forward(pb):
    """Gradients equal torch autograd of the forward restated in torch ops, and that restatement's
    output equals the oracle's own forward (exact pooling, the oracle's selection lists)."""
    q, k, v, g, dout = _bwd_inputs(pb, 71)
    kc = O.pool(pb, k, exact=True)
    vc = O.pool(pb, v, exact=True)
    fwd = O.sparse_attn(pb, q, k, v, g, pooled=(kc, vc))
    leaves = _leaves(q, k, v, g)
    out = _torch_path(pb, *leaves, fwd.idx)
    np.testing.assert_allclose(out.detach().numpy(), fwd.out, rtol=0, atol=1e-12)
    (out * torch.from_numpy(dout)).sum().backward()
    gr = O.backward(pb, q, k, v, g, fwd.idx, dout, kc=kc, vc=vc)
    for name, mine, ref in zip(["dq", "dk", "dv", "dgates"], [gr.dq, gr.dk, gr.dv, gr.dgates],
                               leaves):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=0, atol=1e-11, err_msg=name)


def test_bwd_directional_finite_differences():
    """<grad, u> equals the central difference of <dout, out> along a random direction u of all
    four inputs at once (no autograd anywhere)."""
    pb = O.Problem(246, 2, 16, 32, 3, forced=1, grid_h=10, grid_w=12, special=3, win_h=4)
    q, k, v, g, dout = _bwd_inputs(pb, 83)
    fwd = O.sparse_attn(pb, q, k, v, g, pooled=(O.pool(pb, k, exact=True), O.pool(pb, v, True)))
    gr, _, _ = _bwd(pb, q, k, v, g, fwd.idx, dout)
    x = [torch.from_numpy(values_of(q)), torch.from_numpy(values_of(k)),
         torch.from_numpy(values_of(v)), torch.from_numpy(g.astype(np.float64))]
    gen = torch.Generator().manual_seed(5)
    u = [torch.randn(a.shape, generator=gen, dtype=torch.float64) for a in x]
    D = torch.from_numpy(dout)
    eps = 1e-5

    def f(sign):
        with torch.no_grad():
            return float((_torch_path(pb, *[a + sign * eps * b for a, b in zip(x, u)], fwd.idx)
                          * D).sum())

    fd = (f(1) - f(-1)) / (2 * eps)
    an = sum(float((torch.from_numpy(m) * b).sum())
             for m, b in zip([gr.dq, gr.dk, gr.dv, gr.dgates], u))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


def test_bwd_selection_over_every_block_equals_library_attention_backward():
    """Gate logits (-inf, +inf) switch the compressed branch off; with every key block selected
    the path is dense attention, so dQ, dK, dV are torch SDPA's own fp64 backward and the gate
    gradients vanish."""
    for pb in [O.Problem(200, 2, 16, 32, 7), O.Problem(200, 2, 16, 32, 5, forced=2)]:
        g = np.zeros((pb.L, pb.H, 2), np.float32)
        g[..., 0], g[..., 1] = -np.inf, np.inf
        q, k, v, g, dout = _bwd_inputs(pb, 91, gates=g)
        idx = np.broadcast_to(np.arange(pb.nb, dtype=np.int32)[::-1], (pb.H, pb.nqb, pb.nb))
        gr, _, _ = _bwd(pb, q, k, v, g, idx, dout)
        tq, tk, tv = [torch.tensor(values_of(a)).permute(1, 0, 2)[None].requires_grad_()
                      for a in (q, k, v)]
        o = F.scaled_dot_product_attention(tq, tk, tv, scale=pb.softmax_scale)
        (o[0].permute(1, 0, 2) * torch.from_numpy(dout)).sum().backward()
        for mine, ref in zip([gr.dq, gr.dk, gr.dv], [tq, tk, tv]):
            np.testing.assert_allclose(mine, ref.grad[0].permute(1, 0, 2).numpy(), rtol=0,
                                       atol=1e-11)
        assert np.all(gr.dgates == 0.0)


@pytest.mark.parametrize("L", [256, 200])
def test_bwd_compressed_branch_equals_library_attention_over_pooled_keys(L):
    """Gate logits (+inf, -inf) leave the compressed branch alone: dense attention of every query
    over the block means, whose gradient reaches each token through the mean (torch autograd
    of SDPA over torch-pooled K/V; a ragged last block is the mean of its own tokens)."""
    pb = O.Problem(L, 2, 16, 32, 2)
    g = np.zeros((pb.L, pb.H, 2), np.float32)
    g[..., 0], g[..., 1] = np.inf, -np.inf
    q, k, v, g, dout = _bwd_inputs(pb, 97, gates=g)
    idx = np.zeros((pb.H, pb.nqb, pb.nsel), np.int32) + np.arange(pb.nsel, dtype=np.int32)
    gr, _, _ = _bwd(pb, q, k, v, g, idx, dout)
    tq, tk, tv = [torch.tensor(values_of(a), requires_grad=True) for a in (q, k, v)]
    kc = torch.stack([c.mean(0) for c in torch.split(tk, pb.block)])
    vc = torch.stack([c.mean(0) for c in torch.split(tv, pb.block)])
    o = F.scaled_dot_product_attention(tq.permute(1, 0, 2)[None], kc.permute(1, 0, 2)[None],
                                       vc.permute(1, 0, 2)[None], scale=pb.softmax_scale)
    (o[0].permute(1, 0, 2) * torch.from_numpy(dout)).sum().backward()
    for mine, ref in zip([gr.dq, gr.dk, gr.dv], [tq, tk, tv]):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=0, atol=1e-11)


def test_bwd_key_gradients_sum_to_zero_and_value_gradients_conserve_mass():
    """Softmax weights sum to one in both branches and pooling keeps sums, so per head the key
    gradients sum to zero over all tokens (a common shift of every key changes nothing) and the
    value gradients sum to sum_r (sigmoid(g0) + sigmoid(g1)) dout_r."""
    pb = O.Problem(246, 3, 16, 32, 3, forced=1, grid_h=10, grid_w=12, special=3, win_h=4)
    q, k, v, g, dout = _bwd_inputs(pb, 101)
    fwd = O.sparse_attn(pb, q, k, v, g)
    gr, _, _ = _bwd(pb, q, k, v, g, fwd.idx, dout)
    assert np.abs(gr.dk.sum(0)).max() < 1e-11
    s = 1 / (1 + np.exp(-g.astype(np.float64)))
    np.testing.assert_allclose(gr.dv.sum(0), ((s[..., :1] + s[..., 1:]) * dout).sum(0), rtol=0,
                               atol=1e-11)


def test_bwd_equal_values_leave_no_attention_gradient():
    """When every value row of a head is the same vector w, both branch outputs are w whatever
    the weights: dQ = dK = 0 and the gate gradients are sigmoid'(g) <dout, w>."""
    pb = O.Problem(200, 2, 16, 32, 3, forced=1)
    q, k, _, g, dout = _bwd_inputs(pb, 107)
    w = rand_bits((1, pb.H, pb.d), 109, 1.0)
    v = np.ascontiguousarray(np.broadcast_to(w, (pb.L, pb.H, pb.d)))
    fwd = O.sparse_attn(pb, q, k, v, g)
    gr, _, _ = _bwd(pb, q, k, v, g, fwd.idx, dout)
    assert np.abs(gr.dq).max() < 1e-12 and np.abs(gr.dk).max() < 1e-12
    s = 1 / (1 + np.exp(-g.astype(np.float64)))
    yw = (dout * values_of(w)).sum(-1)
    np.testing.assert_allclose(gr.dgates, s * (1 - s) * yw[..., None], rtol=0, atol=1e-12)


def test_bwd_rejects_an_out_of_range_index():
    pb = O.Problem(200, 1, 16, 32, 2)
    q, k, v, g, dout = _bwd_inputs(pb, 113)
    idx = np.zeros((pb.H, pb.nqb, pb.nsel), np.int32)
    idx[0, 1, 1] = pb.nb
    with pytest.raises(AssertionError, match="-3"):
        _bwd(pb, q, k, v, g, idx, dout)


def test_bwd_sampled_query_blocks_equal_full_run():
    """dq and dgates of a row depend only on that row: the backward of a sample of query blocks
    (in any order, the partial last one included) gives exactly the full run's rows."""
    pb = O.Problem(246, 2, 16, 32, 3, forced=1, grid_h=10, grid_w=12, special=3, win_h=4)
    q, k, v, g, dout = _bwd_inputs(pb, 117)
    fwd = O.sparse_attn(pb, q, k, v, g)
    full, kc, vc = _bwd(pb, q, k, v, g, fwd.idx, dout)
    qb = [3, 0, 2]  # nqb = 4; block 3 holds the last 54 rows
    rows = pb.rows_of(qb)
    part = O.backward(pb, q, k, v, g, np.ascontiguousarray(fwd.idx[:, qb]), dout[rows], kc=kc,
                      vc=vc, qblocks=qb)
    assert part.dk is None and part.dv is None
    np.testing.assert_array_equal(part.dq, full.dq[rows])
    np.testing.assert_array_equal(part.dgates, full.dgates[rows])


def test_bwd_random_configurations_equal_autograd():
    """Seeded small configurations across every axis at once (block size, top-k, forced blocks,
    1-D or 2-D geometry with special tokens and cut windows, ragged tails, scale): the oracle's
    gradients equal torch autograd of the torch restatement of the forward."""
    rng = np.random.default_rng(2024)
    for trial in range(8):
        b = int(rng.choice([8, 16, 32]))
        if trial % 2:  # 2-D windows
            wh = int(rng.choice([w for w in (1, 2, 4, 8) if b % w == 0]))
            gh, gw = int(rng.integers(2, 9)), int(rng.integers(2, 12))
            special = int(rng.integers(0, min(b, 6) + 1))
            N = int(rng.integers(1, 4))
            geo = dict(grid_h=gh, grid_w=gw, special=special, win_h=wh)
            L = N * (special + gh * gw)
        else:
            geo = {}
            L = int(rng.integers(20, 200))
        nb = O.Problem(L, 1, 16, b, 1, **geo).nb
        forced = int(rng.integers(0, min(3, nb - 1) + 1)) if nb > 1 else 0
        k = int(rng.integers(1, nb - forced + 1))
        H = int(rng.integers(1, 3))
        scale = None if trial % 3 else float(rng.uniform(0.05, 0.4))
        pb = O.Problem(L, H, 16, b, k, qblock=int(rng.choice([16, 32, 64])), scale=scale,
                       forced=forced, **geo)
        q, kk, v, g, dout = _bwd_inputs(pb, 300 + trial)
        kc = O.pool(pb, kk, exact=True)
        vc = O.pool(pb, v, exact=True)
        fwd = O.sparse_attn(pb, q, kk, v, g, pooled=(kc, vc))
        leaves = _leaves(q, kk, v, g)
        out = _torch_path(pb, *leaves, fwd.idx)
        np.testing.assert_allclose(out.detach().numpy(), fwd.out, rtol=0, atol=1e-12)
        (out * torch.from_numpy(dout)).sum().backward()
        gr = O.backward(pb, q, kk, v, g, fwd.idx, dout, kc=kc, vc=vc)
        for name, mine, ref in zip(["dq", "dk", "dv", "dgates"],
                                   [gr.dq, gr.dk, gr.dv, gr.dgates], leaves):
            np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=0, atol=1e-11,
                                       err_msg=f"trial {trial}: {name} {pb}")


def test_bwd_keys_equal_autograd_rows_of_the_listed_blocks():
    """s3r_ref_bwd_keys: dk and dv of one head for the tokens of a few key blocks (the first, the
    ragged last, one in the middle) equal torch autograd of the torch restatement of the forward
    on those tokens, on 1-D blocks, with forced blocks, and on 2-D windows with special tokens;
    the rows past a block's token count are zero."""
    for pb, seed in [(O.Problem(200, 2, 16, 32, 3), 401),
                     (O.Problem(190, 2, 16, 16, 2, forced=2), 402),
                     (O.Problem(2 * (3 + 6 * 10), 2, 16, 16, 3, forced=1, grid_h=6, grid_w=10,
                                special=3, win_h=2), 403)]:
        q, kk, v, g, dout = _bwd_inputs(pb, seed)
        kc = O.pool(pb, kk, exact=True)
        vc = O.pool(pb, v, exact=True)
        fwd = O.sparse_attn(pb, q, kk, v, g, pooled=(kc, vc))
        leaves = _leaves(q, kk, v, g)
        out = _torch_path(pb, *leaves, fwd.idx)
        (out * torch.from_numpy(dout)).sum().backward()
        blocks = [0, pb.nb - 1, pb.nb // 2]
        for h in range(pb.H):
            dk, dv = O.backward_keys(pb, q, kk, v, g, fwd.idx, dout, h, blocks, kc=kc, vc=vc)
            for a, j in enumerate(blocks):
                t = pb.block_tokens(j)
                np.testing.assert_allclose(dk[a, :t.size], leaves[1].grad.numpy()[t, h], rtol=0,
                                           atol=1e-11, err_msg=f"{pb} head {h} block {j}")
                np.testing.assert_allclose(dv[a, :t.size], leaves[2].grad.numpy()[t, h], rtol=0,
                                           atol=1e-11, err_msg=f"{pb} head {h} block {j}")
                assert not dk[a, t.size:].any() and not dv[a, t.size:].any()
