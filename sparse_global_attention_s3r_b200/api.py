"""torch-tensor front end of libs3r.so: shape checks, output allocation, pointer marshalling.

Every step of the computation runs in the library's CUDA kernels; torch only provides device
memory and the current stream. All tensors must be CUDA tensors of the current device, dense and
contiguous, with the layouts of include/s3r.h:

    q, k, v      [L, H, 64] bf16          gates  [L, H, 2] fp32
    k_cmp, v_cmp [nb, H, 64] bf16         lse    [H, L] fp32
    o_cmp, o_sel [L, H, 64] fp32          scores [H, nqb, nb] fp32
    idx          [H, nqb, forced + topk] int32
    out, dout    [L, H, 64] bf16
    dq, dk, dv   [L, H, 64] fp32          dgates [L, H, 2] fp32
nb counts the key blocks of the configured geometry (Config.nb), nqb = ceil(L / 64).
"""
from __future__ import annotations

import ctypes
import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _lib

QBLOCK = 64


@dataclass(frozen=True)
class Config:
    """Sizes of one call: L tokens (N views x P tokens), H heads, d, block size b, top-k.

    forced: leading key blocks kept in every selection list (VGGT's reference frame: with P
    tokens per view, ceil(P / b)); the top-k then picks topk more among the other blocks.
    grid_h, grid_w, special, win_h: 2-D windows (grid_h > 0). The sequence is L / P views of
    P = special + grid_h * grid_w tokens; key blocks are each view's special tokens, then
    win_h x (block / win_h) windows of its patch grid.
    save_for_backward: the forward keeps in its workspace what the backward needs, and a backward
    call with the same config and workspace skips recomputing the forward.
    nvtx: the whole-path calls push one NVTX range per stage (s3r.pool, s3r.cmp, ...)."""

    L: int
    H: int
    d: int = 64
    block: int = 64
    topk: int = 16
    scale: Optional[float] = None  # None -> 1/sqrt(d)
    debug_checks: bool = False
    test_timeout: bool = False  # testing only: exercise the bounded-wait timeout path
    single_kernel: bool = False  # topk <= 32: compressed branch, top-k and selection in one kernel
    forced: int = 0
    grid_h: int = 0
    grid_w: int = 0
    special: int = 0
    win_h: int = 0
    save_for_backward: bool = False
    nvtx: bool = False  # one NVTX range per stage of the whole-path calls, for profilers

    @property
    def nsel(self) -> int:
        """Selection list length: forced blocks, then the top-k."""
        return self.forced + self.topk

    @property
    def nb(self) -> int:
        """Key blocks, as the library counts them (0 for invalid sizes)."""
        return int(_lib.load().s3r_num_key_blocks(ctypes.byref(self.params())))

    @property
    def nqb(self) -> int:
        return -(-self.L // QBLOCK)

    def params(self, dev_status: Optional[torch.Tensor] = None, stage_events=None) -> _lib.Params:
        return _lib.Params(self.L, self.H, self.d, self.block, QBLOCK, self.topk,
                           0.0 if self.scale is None else float(self.scale),
                           (_lib.S3R_FLAG_DEBUG_CHECKS if self.debug_checks else 0)
                           | (_lib.S3R_FLAG_TEST_TIMEOUT if self.test_timeout else 0)
                           | (_lib.S3R_FLAG_SINGLE_KERNEL if self.single_kernel else 0)
                           | (_lib.S3R_FLAG_SAVE_FOR_BWD if self.save_for_backward else 0)
                           | (_lib.S3R_FLAG_NVTX if self.nvtx else 0),
                           self.forced, self.grid_h, self.grid_w, self.special, self.win_h,
                           None if dev_status is None else dev_status.data_ptr(),
                           None if stage_events is None else ctypes.addressof(stage_events))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t: torch.Tensor, name: str, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} contiguous={t.is_contiguous()}")


def _lhd(cfg: Config):
    return (cfg.L, cfg.H, cfg.d)


def compress_kv(cfg: Config, k: torch.Tensor, v: torch.Tensor,
                dev_status: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    _need(k, "k", _lhd(cfg), torch.bfloat16)
    _need(v, "v", _lhd(cfg), torch.bfloat16)
    kc = torch.empty((cfg.nb, cfg.H, cfg.d), dtype=torch.bfloat16, device=k.device)
    vc = torch.empty_like(kc)
    p = cfg.params(dev_status)
    _lib.call("s3r_compress_kv", ctypes.byref(p), _ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _stream())
    return kc, vc


def cmp_attn_and_score(cfg: Config, q: torch.Tensor, kc: torch.Tensor, vc: torch.Tensor,
                       dev_status: Optional[torch.Tensor] = None):
    """-> (o_cmp [L,H,d] fp32, lse [H,L] fp32, scores [H,nqb,nb] fp32)"""
    _need(q, "q", _lhd(cfg), torch.bfloat16)
    _need(kc, "k_cmp", (cfg.nb, cfg.H, cfg.d), torch.bfloat16)
    _need(vc, "v_cmp", (cfg.nb, cfg.H, cfg.d), torch.bfloat16)
    o = torch.empty(_lhd(cfg), dtype=torch.float32, device=q.device)
    lse = torch.empty((cfg.H, cfg.L), dtype=torch.float32, device=q.device)
    scores = torch.empty((cfg.H, cfg.nqb, cfg.nb), dtype=torch.float32, device=q.device)
    p = cfg.params(dev_status)
    _lib.call("s3r_cmp_attn_and_score", ctypes.byref(p), _ptr(q), _ptr(kc), _ptr(vc), _ptr(o),
              _ptr(lse), _ptr(scores), _stream())
    return o, lse, scores


def topk_blocks(cfg: Config, scores: torch.Tensor,
                dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    _need(scores, "scores", (cfg.H, cfg.nqb, cfg.nb), torch.float32)
    idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=scores.device)
    p = cfg.params(dev_status)
    _lib.call("s3r_topk_blocks", ctypes.byref(p), _ptr(scores), _ptr(idx), _stream())
    return idx


def sel_attn(cfg: Config, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
             dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, _lhd(cfg), torch.bfloat16)
    _need(idx, "idx", (cfg.H, cfg.nqb, cfg.nsel), torch.int32)
    o = torch.empty(_lhd(cfg), dtype=torch.float32, device=q.device)
    p = cfg.params(dev_status)
    _lib.call("s3r_sel_attn", ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(o),
              _stream())
    return o


def gate_combine(cfg: Config, o_cmp: torch.Tensor, o_sel: torch.Tensor,
                 gates: torch.Tensor) -> torch.Tensor:
    _need(o_cmp, "o_cmp", _lhd(cfg), torch.float32)
    _need(o_sel, "o_sel", _lhd(cfg), torch.float32)
    _need(gates, "gates", (cfg.L, cfg.H, 2), torch.float32)
    out = torch.empty(_lhd(cfg), dtype=torch.bfloat16, device=o_cmp.device)
    p = cfg.params()
    _lib.call("s3r_gate_combine", ctypes.byref(p), _ptr(o_cmp), _ptr(o_sel), _ptr(gates),
              _ptr(out), _stream())
    return out


def workspace_bytes(cfg: Config) -> int:
    p = cfg.params()
    n = int(_lib.load().s3r_workspace_bytes(ctypes.byref(p)))
    if n == 0:
        raise _lib.S3RError("s3r_workspace_bytes", _lib.S3R_ERR_INVALID_ARG)
    return n


def alloc_workspace(cfg: Config, device=None) -> torch.Tensor:
    n = workspace_bytes(cfg)
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=device or torch.cuda.current_device())


class StageEvents:
    """CUDA events that s3r_sparse_attn_fwd (S3R_NUM_STAGES + 1) or, with stages=
    _lib.BWD_STAGES, s3r_sparse_attn_bwd (S3R_NUM_BWD_STAGES + 1) records at its stage
    boundaries."""

    def __init__(self, stages=_lib.STAGES):
        self.stages = stages
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)]
        for e in self.events:  # torch creates the underlying event on first record
            e.record()
        self.handles = (ctypes.c_void_p * len(self.events))(
            *[e.cuda_event for e in self.events])

    def stage_ms(self) -> dict:
        """Milliseconds of each stage of the last recorded call (events must have completed)."""
        return {n: self.events[i].elapsed_time(self.events[i + 1])
                for i, n in enumerate(self.stages)}


def sparse_attn_fwd(cfg: Config, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    gates: torch.Tensor, workspace: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, idx_out: Optional[torch.Tensor] = None,
                    dev_status: Optional[torch.Tensor] = None,
                    stage_events: Optional[StageEvents] = None) -> torch.Tensor:
    """The whole path in one library call; returns out [L,H,d] bf16 (idx written if given)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, _lhd(cfg), torch.bfloat16)
    _need(gates, "gates", (cfg.L, cfg.H, 2), torch.float32)
    if workspace is None:
        workspace = alloc_workspace(cfg, q.device)
    if out is None:
        out = torch.empty(_lhd(cfg), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", _lhd(cfg), torch.bfloat16)
    if idx_out is not None:
        _need(idx_out, "idx_out", (cfg.H, cfg.nqb, cfg.nsel), torch.int32)
    p = cfg.params(dev_status, None if stage_events is None else stage_events.handles)
    _lib.call("s3r_sparse_attn_fwd", ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
              _ptr(out), _ptr(idx_out), _ptr(workspace), workspace.numel(), _stream())
    return out


def sparse_attn_fwd_static(cfg: Config, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                           gates: torch.Tensor, out: Optional[torch.Tensor] = None,
                           idx_out: Optional[torch.Tensor] = None,
                           dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole path without a workspace argument: the library's built-in scratch array is used
    (sizes up to S3R_STATIC_WORKSPACE_BYTES of workspace; see include/s3r.h). The entry point
    reports device-side conditions only through a caller's status word: pass dev_status (one
    int32 on the device, read it with read_device_status), or one is allocated here."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _need(t, n, _lhd(cfg), torch.bfloat16)
    _need(gates, "gates", (cfg.L, cfg.H, 2), torch.float32)
    if out is None:
        out = torch.empty(_lhd(cfg), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", _lhd(cfg), torch.bfloat16)
    if idx_out is not None:
        _need(idx_out, "idx_out", (cfg.H, cfg.nqb, cfg.nsel), torch.int32)
    if dev_status is None:
        dev_status = torch.zeros(1, dtype=torch.int32, device=q.device)
    p = cfg.params(dev_status)
    _lib.call("s3r_sparse_attn_fwd_static", ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
              _ptr(gates), _ptr(out), _ptr(idx_out), _stream())
    return out


def bwd_workspace_bytes(cfg: Config) -> int:
    p = cfg.params()
    n = int(_lib.load().s3r_bwd_workspace_bytes(ctypes.byref(p)))
    if n == 0:
        raise _lib.S3RError("s3r_bwd_workspace_bytes", _lib.S3R_ERR_INVALID_ARG)
    return n


def sparse_attn_bwd(cfg: Config, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                    gates: torch.Tensor, idx: torch.Tensor, dout: torch.Tensor,
                    workspace: Optional[torch.Tensor] = None,
                    dev_status: Optional[torch.Tensor] = None,
                    stage_events: Optional[StageEvents] = None, grads=None):
    """Gradients of the whole path for the upstream gradient dout, with the selection lists idx
    (the forward's idx_out) held fixed: returns dq, dk, dv [L,H,d] fp32 and dgates [L,H,2] fp32.

    grads: optional preallocated (dq, dk, dv, dgates) to write into; stage_events: a
    StageEvents(_lib.BWD_STAGES) that the call records at its stage boundaries. With
    cfg.save_for_backward, workspace must be the one the forward call used (allocate
    bwd_workspace_bytes(cfg) bytes and pass it to both)."""
    for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, n, _lhd(cfg), torch.bfloat16)
    _need(gates, "gates", (cfg.L, cfg.H, 2), torch.float32)
    _need(idx, "idx", (cfg.H, cfg.nqb, cfg.nsel), torch.int32)
    if workspace is None:
        if cfg.save_for_backward:
            raise ValueError("save_for_backward: pass the forward call's workspace")
        workspace = torch.empty(bwd_workspace_bytes(cfg), dtype=torch.uint8, device=q.device)
    if grads is None:
        grads = (*(torch.empty(_lhd(cfg), dtype=torch.float32, device=q.device) for _ in range(3)),
                 torch.empty((cfg.L, cfg.H, 2), dtype=torch.float32, device=q.device))
    dq, dk, dv, dgates = grads
    for n, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, n, _lhd(cfg), torch.float32)
    _need(dgates, "dgates", (cfg.L, cfg.H, 2), torch.float32)
    p = cfg.params(dev_status, None if stage_events is None else stage_events.handles)
    _lib.call("s3r_sparse_attn_bwd", ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(gates),
              _ptr(idx), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgates), _ptr(workspace),
              workspace.numel(), _stream())
    return dq, dk, dv, dgates


class SparseAttentionFunction(torch.autograd.Function):
    """autograd wrapper: forward = sparse_attn_fwd (bf16 out), backward = sparse_attn_bwd.

    Gradients are returned in the inputs' dtypes (bf16 for q, k, v; fp32 for the gate logits).
    The top-k selection passes no gradient. The forward runs with save_for_backward and keeps
    its workspace until the backward, which then does not recompute the forward. That is
    bwd_workspace_bytes(cfg) bytes, about 816 per (token, head): O_cmp and O_sel in fp32, the
    slot-order K/V copies, the lse and the backward's scratch."""

    @staticmethod
    def forward(ctx, q, k, v, gates, cfg: Config):
        cfg = dataclasses.replace(cfg, save_for_backward=True, single_kernel=False)
        idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=q.device)
        ws = torch.empty(bwd_workspace_bytes(cfg), dtype=torch.uint8, device=q.device)
        out = sparse_attn_fwd(cfg, q, k, v, gates, workspace=ws, idx_out=idx)
        ctx.cfg = cfg
        ctx.ws = ws
        ctx.save_for_backward(q, k, v, gates, idx)
        ctx.mark_non_differentiable(idx)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, gates, idx = ctx.saved_tensors
        dq, dk, dv, dg = sparse_attn_bwd(ctx.cfg, q, k, v, gates, idx,
                                         dout.to(torch.bfloat16).contiguous(), workspace=ctx.ws)
        ctx.ws = None
        return dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), dg, None


def read_device_status(word: torch.Tensor) -> int:
    """Synchronise the current stream, return and clear the device status word."""
    v = ctypes.c_uint32(0)
    st = _lib.load().s3r_read_device_status(_ptr(word), _stream(), ctypes.byref(v))
    if st not in (_lib.S3R_OK, _lib.S3R_ERR_TIMEOUT):
        _lib.check("s3r_read_device_status", st)
    return int(v.value)


class SparseAttention:
    """Reusable caller of the fused path: owns its workspace and output buffers on one device.

    ``__call__`` takes device tensors. ``from_host`` takes pinned host tensors, copies them in,
    runs the path and copies the output (and indices) back: the end-to-end use.
    """

    def __init__(self, cfg: Config, device=None):
        self.cfg = cfg
        self.device = torch.device(device or "cuda")
        self.workspace = alloc_workspace(cfg, self.device)
        self.out = torch.empty(_lhd(cfg), dtype=torch.bfloat16, device=self.device)
        self.idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=self.device)
        self._dev_in = None

    def __call__(self, q, k, v, gates) -> torch.Tensor:
        return sparse_attn_fwd(self.cfg, q, k, v, gates, self.workspace, self.out, self.idx)

    def from_host(self, q, k, v, gates, out_host: torch.Tensor) -> torch.Tensor:
        if self._dev_in is None:
            self._dev_in = [torch.empty_like(t, device=self.device) for t in (q, k, v, gates)]
        for dst, src in zip(self._dev_in, (q, k, v, gates)):
            dst.copy_(src, non_blocking=True)
        self(*self._dev_in)
        out_host.copy_(self.out, non_blocking=True)
        return out_host


class HostPipeline:
    """The fused path over a stream of independent steps whose inputs live in pinned host memory.

    ``submit`` enqueues one step: its inputs are copied in on a copy-in stream, the path runs on
    the caller's current stream, and the output is copied back on a copy-out stream. Two sets of
    device inputs and outputs alternate, so the copy-in of step i+1 and the copy-out of step i-1
    overlap the kernels of step i; each step still moves all of its inputs in and its output out.
    Everything is asynchronous: ``synchronize`` waits for every submitted step, after which the
    host outputs may be read. A host output buffer must not be reused before that.
    """

    def __init__(self, cfg: Config, device=None):
        self.cfg = cfg
        self.device = torch.device(device or "cuda")
        self.workspace = alloc_workspace(cfg, self.device)
        self.idx = torch.empty((cfg.H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=self.device)
        lhd = _lhd(cfg)
        self.ins = [[torch.empty(lhd, dtype=torch.bfloat16, device=self.device) for _ in range(3)]
                    + [torch.empty((cfg.L, cfg.H, 2), dtype=torch.float32, device=self.device)]
                    for _ in range(2)]
        self.outs = [torch.empty(lhd, dtype=torch.bfloat16, device=self.device) for _ in range(2)]
        self.copy_in = torch.cuda.Stream(self.device)
        self.copy_out = torch.cuda.Stream(self.device)
        self.ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of the slot are on device
        self.ev_done = [torch.cuda.Event() for _ in range(2)]  # the slot's kernels have finished
        self.ev_out = [torch.cuda.Event() for _ in range(2)]   # the slot's output is on the host
        self.steps = 0

    def submit(self, q, k, v, gates, out_host: torch.Tensor, after: torch.cuda.Event = None):
        """Enqueue one step (q, k, v bf16 and gates fp32, pinned host tensors) writing out_host.
        ``after``: an event the copy-in of this step waits for (e.g. a timing start)."""
        i = self.steps % 2
        compute = torch.cuda.current_stream(self.device)
        with torch.cuda.stream(self.copy_in):
            if after is not None:
                self.copy_in.wait_event(after)
            if self.steps >= 2:  # step n-2 has finished reading this slot's inputs
                self.copy_in.wait_event(self.ev_done[i])
            for dst, src in zip(self.ins[i], (q, k, v, gates)):
                dst.copy_(src, non_blocking=True)
            self.ev_in[i].record(self.copy_in)
        compute.wait_event(self.ev_in[i])
        if self.steps >= 2:  # step n-2's output has left this slot
            compute.wait_event(self.ev_out[i])
        sparse_attn_fwd(self.cfg, *self.ins[i], self.workspace, self.outs[i], self.idx)
        self.ev_done[i].record(compute)
        with torch.cuda.stream(self.copy_out):
            self.copy_out.wait_event(self.ev_done[i])
            out_host.copy_(self.outs[i], non_blocking=True)
            self.ev_out[i].record(self.copy_out)
        self.steps += 1
        return out_host

    def synchronize(self) -> None:
        self.copy_out.synchronize()
        torch.cuda.current_stream(self.device).synchronize()
