"""numpy front-end of the fp64 CPU oracle (oracle/s3r_oracle.c).

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only tests/, the smoke check and the benchmark's
CPU-baseline leg import this module. It shares nothing with the CUDA library: it loads its own
shared object built from oracle/s3r_oracle.c.

Method: the gist.science summary of "Speed3R: Sparse Feed-forward 3D Reconstruction Models",
"Technische samenvatting" -> "Methodologie" §1 (compression branch with average pooling and a score
matrix; selection branch on the top-k blocks) and §2 (gated aggregation). The readings taken where
the pages are silent are listed in oracle/s3r_oracle.c.

bf16 tensors travel as numpy uint16 arrays of their bit patterns; use ``bf16_bits`` to obtain
them from a torch bf16 tensor.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_LIB = None


class _Params(ctypes.Structure):
    _fields_ = [
        ("L", ctypes.c_int64),
        ("H", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("qblock", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("scale", ctypes.c_double),
        ("exact_pool", ctypes.c_int32),
        ("threads", ctypes.c_int32),
        ("forced", ctypes.c_int32),
        ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32),
        ("special", ctypes.c_int32),
        ("win_h", ctypes.c_int32),
    ]


def lib():
    """Load (building first if needed) the oracle shared library.

    S3R_ORACLE_LIB, when set, names another build of oracle/s3r_oracle.c to load instead; the
    mutation test uses it to run the pins against deliberately broken copies.
    """
    global _LIB
    if _LIB is None:
        path = os.environ.get("S3R_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        p = ctypes.c_void_p
        L.s3r_ref_hardware_threads.restype = ctypes.c_int
        L.s3r_ref_round_bf16.restype = ctypes.c_double
        L.s3r_ref_round_bf16.argtypes = [ctypes.c_double]
        for name, args in {
            "s3r_ref_pool": [p, p, p],
            "s3r_ref_cmp": [p, p, p, p, p, ctypes.c_int64, p, p, p],
            "s3r_ref_topk": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, p, p, p],
            "s3r_ref_sel": [p, p, p, p, p, ctypes.c_int64, p, p],
            "s3r_ref_combine": [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, p, p, p, p],
            "s3r_ref_block_tokens": [p, ctypes.c_int64, p],
            "s3r_ref_bwd": [p, p, p, p, p, p, p, p, p, ctypes.c_int64, p, p, p, p, p],
            "s3r_ref_bwd_keys": [p, p, p, p, p, p, p, p, ctypes.c_int32, p, ctypes.c_int64, p, p,
                                 p],
        }.items():
            fn = getattr(L, name)
            fn.restype = ctypes.c_int
            fn.argtypes = args
        L.s3r_ref_num_blocks.restype = ctypes.c_int64
        L.s3r_ref_num_blocks.argtypes = [ctypes.c_void_p]
        L.s3r_ref_block_tokens.restype = ctypes.c_int64
        _LIB = L
    return _LIB


@dataclass
class Problem:
    """Sizes of one sparse-attention call. Blocks run over the flattened sequence of L tokens."""

    L: int
    H: int
    d: int
    block: int
    topk: int
    qblock: int = 64
    scale: Optional[float] = None  # None -> 1/sqrt(d)
    forced: int = 0  # leading key blocks kept in every selection list (VGGT reference frame)
    # 2-D windows (grid_h > 0): views of `special` tokens + a grid_h x grid_w patch grid, key
    # blocks = the special tokens of a view, then win_h x (block / win_h) windows of its grid
    grid_h: int = 0
    grid_w: int = 0
    special: int = 0
    win_h: int = 0

    @property
    def nb(self) -> int:
        if self.grid_h == 0:
            return -(-self.L // self.block)
        n = lib().s3r_ref_num_blocks(ctypes.byref(_params(self)))
        assert n > 0, "invalid 2-D geometry"
        return int(n)

    def block_tokens(self, j: int) -> np.ndarray:
        """Tokens of key block j, ascending."""
        out = np.empty(self.block, np.int64)
        n = lib().s3r_ref_block_tokens(ctypes.byref(_params(self)), j, _ptr(out))
        assert n >= 0, n
        return out[:n].copy()

    @property
    def nqb(self) -> int:
        return -(-self.L // self.qblock)

    @property
    def nsel(self) -> int:
        """Length of a selection list: the forced blocks, then the top-k."""
        return self.forced + self.topk

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    def rows_of(self, qblocks: Optional[Sequence[int]]) -> np.ndarray:
        """Sequence rows of the chosen query blocks, concatenated in list order."""
        if qblocks is None:
            return np.arange(self.L, dtype=np.int64)
        parts = [np.arange(i * self.qblock, min((i + 1) * self.qblock, self.L)) for i in qblocks]
        return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def _params(pb: Problem, exact_pool: bool = False, threads: int = 0) -> _Params:
    return _Params(pb.L, pb.H, pb.d, pb.block, pb.qblock, pb.topk, pb.softmax_scale,
                   1 if exact_pool else 0, threads, pb.forced, pb.grid_h, pb.grid_w, pb.special,
                   pb.win_h)


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _qb_array(qblocks):
    if qblocks is None:
        return None, 0
    a = np.ascontiguousarray(np.asarray(qblocks, dtype=np.int64))
    return a, a.size


def bf16_bits(t) -> np.ndarray:
    """uint16 bit patterns of a torch bf16 tensor (any device), as a contiguous numpy array."""
    import torch

    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def round_bf16(x: float) -> float:
    return lib().s3r_ref_round_bf16(float(x))


def hardware_threads() -> int:
    return lib().s3r_ref_hardware_threads()


def pool(pb: Problem, x_bits: np.ndarray, exact: bool = False, threads: int = 0) -> np.ndarray:
    """Block means [nb, H, d] of x [L, H, d] (bf16 bits); rounded to bf16 unless exact."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    assert x_bits.shape == (pb.L, pb.H, pb.d)
    out = np.empty((pb.nb, pb.H, pb.d), np.float64)
    rc = lib().s3r_ref_pool(ctypes.byref(_params(pb, exact, threads)), _ptr(x_bits), _ptr(out))
    assert rc == 0, rc
    return out


def cmp_attn(pb: Problem, q_bits, kc, vc, qblocks=None, threads: int = 0):
    """Compression branch over the chosen query blocks: (lse [H,R], o_cmp [R,H,d], scores [H,nq,nb])."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kc = np.ascontiguousarray(kc, dtype=np.float64)
    vc = np.ascontiguousarray(vc, dtype=np.float64)
    qa, nq = _qb_array(qblocks)
    if qa is None:
        nq = pb.nqb
    R = pb.rows_of(qblocks).size
    lse = np.empty((pb.H, R), np.float64)
    o = np.empty((R, pb.H, pb.d), np.float64)
    sc = np.empty((pb.H, nq, pb.nb), np.float64)
    rc = lib().s3r_ref_cmp(ctypes.byref(_params(pb, threads=threads)), _ptr(q_bits), _ptr(kc),
                           _ptr(vc), None if qa is None else _ptr(qa), nq, _ptr(lse), _ptr(o),
                           _ptr(sc))
    assert rc == 0, rc
    return lse, o, sc


def topk(scores: np.ndarray, k: int, forced: int = 0):
    """Selection lists along the last axis: (idx int32 [..., forced + k], gap [...]).

    The lists open with blocks 0 .. forced-1; the top-k (ties -> lower index first) ranks only the
    other blocks, and gap is the k-th minus the (k+1)-th of those."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    lead = s.shape[:-1]
    n = s.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    idx = np.empty(lead + (forced + k,), np.int32)
    gap = np.empty(lead, np.float64)
    rc = lib().s3r_ref_topk(rows, n, k, forced, _ptr(s), _ptr(idx), _ptr(gap))
    assert rc == 0, rc
    return idx, gap


def sel_attn(pb: Problem, q_bits, k_bits, v_bits, idx, qblocks=None, threads: int = 0):
    """Selection branch over the chosen query blocks with the given idx [H, nq, forced + topk]."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    qa, nq = _qb_array(qblocks)
    if qa is None:
        nq = pb.nqb
    assert idx.shape == (pb.H, nq, pb.nsel), idx.shape
    R = pb.rows_of(qblocks).size
    o = np.empty((R, pb.H, pb.d), np.float64)
    rc = lib().s3r_ref_sel(ctypes.byref(_params(pb, threads=threads)), _ptr(q_bits), _ptr(k_bits),
                           _ptr(v_bits), None if qa is None else _ptr(qa), nq, _ptr(idx), _ptr(o))
    assert rc == 0, rc
    return o


def combine(o_cmp, o_sel, gates) -> np.ndarray:
    """sigmoid(g0) * o_cmp + sigmoid(g1) * o_sel; gates fp32 [R, H, 2]."""
    o_cmp = np.ascontiguousarray(o_cmp, dtype=np.float64)
    o_sel = np.ascontiguousarray(o_sel, dtype=np.float64)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    R, H, d = o_cmp.shape
    out = np.empty_like(o_cmp)
    rc = lib().s3r_ref_combine(R, H, d, _ptr(o_cmp), _ptr(o_sel), _ptr(gates), _ptr(out))
    assert rc == 0, rc
    return out


@dataclass
class Grads:
    dq: np.ndarray      # [R, H, d] (R = L, or the rows of the chosen query blocks)
    dk: Optional[np.ndarray]  # [L, H, d]; None for a sample of query blocks
    dv: Optional[np.ndarray]  # [L, H, d]; None for a sample of query blocks
    dgates: np.ndarray  # [R, H, 2] gradient of the gate logits


def backward(pb: Problem, q_bits, k_bits, v_bits, gates, idx, dout, kc=None, vc=None,
             threads: int = 0, qblocks=None) -> Grads:
    """Gradients of the whole path for the upstream gradient dout (float64).

    The selection lists idx are held fixed, and the bf16 rounding of the pooled K/V is passed
    straight through (each token of block j gets dKc[j] / n_j). kc, vc are the pooled values the
    forward ran on (default: ``pool`` of k, v). With qblocks, only the rows of those query blocks
    are differentiated: idx is [H, len(qblocks), forced + topk] for them, dout [R, H, d] their
    rows in list order, and only dq and dgates (row-local) are returned.
    """
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    if kc is None:
        kc = pool(pb, k_bits, threads=threads)
    if vc is None:
        vc = pool(pb, v_bits, threads=threads)
    kc = np.ascontiguousarray(kc, dtype=np.float64)
    vc = np.ascontiguousarray(vc, dtype=np.float64)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    shape = (pb.L, pb.H, pb.d)
    qa, nq = _qb_array(qblocks)
    if qa is None:
        nq = pb.nqb
    R = pb.rows_of(qblocks).size
    assert q_bits.shape == shape and dout.shape == (R, pb.H, pb.d)
    assert gates.shape == (pb.L, pb.H, 2) and kc.shape == (pb.nb, pb.H, pb.d)
    assert idx.shape == (pb.H, nq, pb.nsel), idx.shape
    full = qa is None
    g = Grads(np.empty((R, pb.H, pb.d)), np.empty(shape) if full else None,
              np.empty(shape) if full else None, np.empty((R, pb.H, 2)))
    rc = lib().s3r_ref_bwd(ctypes.byref(_params(pb, threads=threads)), _ptr(q_bits), _ptr(k_bits),
                           _ptr(v_bits), _ptr(kc), _ptr(vc), _ptr(gates), _ptr(idx),
                           None if full else _ptr(qa), nq, _ptr(dout), _ptr(g.dq),
                           _ptr(g.dk) if full else None, _ptr(g.dv) if full else None,
                           _ptr(g.dgates))
    assert rc == 0, rc
    return g


def backward_keys(pb: Problem, q_bits, k_bits, v_bits, gates, idx, dout, head: int, kblocks,
                  kc=None, vc=None, threads: int = 0):
    """dk, dv of one head for the tokens of the key blocks `kblocks` (float64), the same
    gradients as ``backward`` without forming the other blocks': the compressed branch summed over
    every row, spread over each block's tokens through the pooled mean, plus the selection branch
    of the query blocks whose lists hold the block. idx is the full [H, nqb, forced + topk], dout
    the full [L, H, d]. Returns (dk, dv), each [len(kblocks), block, d]: row u of entry a is the
    u-th token of block kblocks[a] (``Problem.block_tokens`` order); rows past its count are 0."""
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    if kc is None:
        kc = pool(pb, k_bits, threads=threads)
    if vc is None:
        vc = pool(pb, v_bits, threads=threads)
    kc = np.ascontiguousarray(kc, dtype=np.float64)
    vc = np.ascontiguousarray(vc, dtype=np.float64)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    dout = np.ascontiguousarray(dout, dtype=np.float64)
    kb = np.ascontiguousarray(kblocks, dtype=np.int64)
    shape = (pb.L, pb.H, pb.d)
    assert q_bits.shape == shape and dout.shape == shape and gates.shape == (pb.L, pb.H, 2)
    assert idx.shape == (pb.H, pb.nqb, pb.nsel), idx.shape
    dk = np.empty((kb.size, pb.block, pb.d))
    dv = np.empty((kb.size, pb.block, pb.d))
    rc = lib().s3r_ref_bwd_keys(ctypes.byref(_params(pb, threads=threads)), _ptr(q_bits),
                                _ptr(k_bits), _ptr(v_bits), _ptr(kc), _ptr(vc), _ptr(gates),
                                _ptr(idx), int(head), _ptr(kb), kb.size, _ptr(dout), _ptr(dk),
                                _ptr(dv))
    assert rc == 0, rc
    return dk, dv


@dataclass
class Result:
    rows: np.ndarray     # sequence rows covered, [R]
    kc: np.ndarray       # pooled K [nb, H, d]
    vc: np.ndarray       # pooled V [nb, H, d]
    lse: np.ndarray      # [H, R]
    o_cmp: np.ndarray    # [R, H, d]
    scores: np.ndarray   # [H, nq, nb]
    idx: np.ndarray      # [H, nq, forced + topk] the oracle's own selection lists
    gap: np.ndarray      # [H, nq]
    idx_used: np.ndarray  # [H, nq, forced + topk] the indices the selection branch ran on
    o_sel: np.ndarray    # [R, H, d]
    out: np.ndarray      # [R, H, d]


def sparse_attn(pb: Problem, q_bits, k_bits, v_bits, gates, qblocks=None, idx_given=None,
                threads: int = 0, pooled=None) -> Result:
    """The whole path on the chosen query blocks.

    idx_given: if not None, the selection branch runs on these indices instead of the oracle's own
    top-k (the conditional oracle used where near-tied scores make the selected set ambiguous).
    pooled: optional (kc, vc) already computed by ``pool`` for the same K, V.
    """
    if pooled is None:
        kc = pool(pb, k_bits, threads=threads)
        vc = pool(pb, v_bits, threads=threads)
    else:
        kc, vc = pooled
    lse, o_cmp, scores = cmp_attn(pb, q_bits, kc, vc, qblocks, threads)
    idx, gap = topk(scores, pb.topk, pb.forced)
    use = idx if idx_given is None else np.ascontiguousarray(idx_given, np.int32)
    o_sel = sel_attn(pb, q_bits, k_bits, v_bits, use, qblocks, threads)
    rows = pb.rows_of(qblocks)
    g = np.ascontiguousarray(np.asarray(gates, np.float32)[rows])
    out = combine(o_cmp, o_sel, g)
    return Result(rows, kc, vc, lse, o_cmp, scores, idx, gap, use, o_sel, out)
