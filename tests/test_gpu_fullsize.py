"""GPU parity at the workload sizes, through the fused entry point exactly as bench.py calls it.

The oracle cannot run the whole layer at these sizes, so it pools all of K/V and then runs the
whole path on a seeded sample of whole query blocks (scores sum over a block, so the sample is
whole blocks; the ragged last block is always included). The GPU's indices and outputs for those
blocks are compared: indices exact where the oracle's k-th/(k+1)-th gap exceeds 1e-4, every
selected block score-optimal within tau, outputs against the oracle run on the GPU's indices.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from sparse_global_attention_s3r_b200 import api, synth

from parity import check_grad, check_output, check_selection

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = {  # name: (L, H, b, k, seed, sampled query blocks[, 2-D geometry, forced views, single])
    "vggt32": (43968, 16, 64, 16, 1, 64),
    "n100": (137400, 16, 64, 32, 2, 48),
    "n1000": (1374000, 16, 64, 32, 3, 64),
    # top-k = 40: the score matrix is written and the stand-alone top-k selects
    "n1000_k40": (1374000, 16, 64, 40, 6, 32),
    "pi3_b32": (274800, 16, 32, 32, 4000, 24),
    "pi3_b64": (274800, 16, 64, 16, 4001, 24),
    "pi3_b128": (274800, 16, 128, 8, 4002, 24),
    "pi3_b64_all_blocks": (274800, 16, 64, 4294, 4003, 3),  # top-k = nb: dense selection
    # the 1000-view layer with 2-D key windows (5 special tokens + 37 x 37 patches a view, 8 x 8)
    "n1000_windows": (1374000, 16, 64, 32, 3, 32, dict(grid_h=37, grid_w=37, special=5, win_h=8)),
    # VGGT-32 with the reference view forced, through the single fused kernel
    "vggt32_ref_view_single": (43968, 16, 64, 16, 5, 48,
                               dict(grid_h=37, grid_w=37, special=5, win_h=8), 1, True),
}


@pytest.mark.parametrize("name", list(FULL))
def test_fused_path_at_workload_size(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L, H, b, k, seed, nsample, *more = FULL[name]
    geo = more[0] if more else {}
    forced_views = more[1] if len(more) > 1 else 0
    single = more[2] if len(more) > 2 else False
    forced = forced_views * (api.Config(L=L, H=H, block=b, topk=1, **geo).nb // (L // (
        geo["special"] + geo["grid_h"] * geo["grid_w"]))) if forced_views else 0
    dev = torch.device("cuda")
    x = synth.make_inputs(L, H, 64, b, seed, device=dev)
    cfg = api.Config(L=L, H=H, block=b, topk=k, forced=forced, single_kernel=single, **geo)
    sa = api.SparseAttention(cfg, dev)
    out = sa(x.q, x.k, x.v, x.gates)
    torch.cuda.synchronize()

    pb = O.Problem(L, H, 64, b, k, forced=forced, **geo)
    rng = np.random.default_rng(seed)
    blocks = sorted(set(rng.choice(cfg.nqb - 1, size=nsample - 1, replace=False).tolist())
                    | {cfg.nqb - 1})
    rows = pb.rows_of(blocks)
    rows_t = torch.from_numpy(rows).to(dev)
    got_out = out.index_select(0, rows_t).double().cpu().numpy()
    got_idx = sa.idx[:, blocks].cpu().numpy()
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    gates = x.gates.cpu().numpy()
    del x, sa, out
    torch.cuda.empty_cache()

    kc, vc = O.pool(pb, bits[1]), O.pool(pb, bits[2])
    ref = O.sparse_attn(pb, *bits, gates, qblocks=blocks, pooled=(kc, vc))
    stats = check_selection(got_idx, ref.idx, ref.gap, ref.scores, k, forced)
    # conditional oracle: the oracle's compressed branch, its selection run on the GPU's indices
    o_sel = O.sel_attn(pb, *bits, got_idx, qblocks=blocks)
    cond_out = O.combine(ref.o_cmp, o_sel, np.ascontiguousarray(gates[rows]))
    err = check_output(got_out, cond_out)
    print(f"{name}: {stats} {err}")


BWD_FULL = {  # name: (L, H, b, k, seed, sampled query blocks[, 2-D geometry, forced views])
    "n100": (137400, 16, 64, 32, 2, 16),
    "n1000": (1374000, 16, 64, 32, 3, 8),
    "vggt32_ref_windows": (43968, 16, 64, 16, 1, 16,
                           dict(grid_h=37, grid_w=37, special=5, win_h=8), 1),
}
# workloads whose sampled key blocks are also compared element by element (the key side of the
# oracle sums the compressed branch over every row of a head, out of reach at 1000 views)
BWD_KEYS = {"n100", "vggt32_ref_windows"}


@pytest.mark.parametrize("name", list(BWD_FULL))
def test_backward_at_workload_size(name):
    """The backward at the workload sizes, after a save-for-backward forward as bench.py runs it.
    dq and dgates of a row depend only on that row: on a seeded sample of query blocks (the
    ragged last one included) they are compared with the oracle's, on the GPU's own lists, under
    the backward bar. dk and dv sum over every query. Everywhere they are checked by properties
    that hold at any size: per head the key gradients sum to zero, and the value gradients sum to
    sum_r (sigmoid(g0) + sigmoid(g1)) dout_r. Where the oracle's key side is within reach
    (BWD_KEYS) the tokens of a few key blocks (the first, which every forced list holds, the
    ragged last and two seeded ones) are also compared element by element, for two heads."""
    import dataclasses

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L, H, b, k, seed, nsample, *more = BWD_FULL[name]
    geo = more[0] if more else {}
    forced = more[1] * (api.Config(L=L, H=H, block=b, topk=1, **geo).nb // (L // (
        geo["special"] + geo["grid_h"] * geo["grid_w"]))) if len(more) > 1 else 0
    dev = torch.device("cuda")
    x = synth.make_inputs(L, H, 64, b, seed, device=dev)
    cfg = dataclasses.replace(api.Config(L=L, H=H, block=b, topk=k, forced=forced, **geo),
                              save_for_backward=True)
    ws = torch.empty(api.bwd_workspace_bytes(cfg), dtype=torch.uint8, device=dev)
    idx = torch.empty((H, cfg.nqb, cfg.nsel), dtype=torch.int32, device=dev)
    api.sparse_attn_fwd(cfg, x.q, x.k, x.v, x.gates, workspace=ws, idx_out=idx)
    g = torch.Generator(device=dev).manual_seed(seed + 7)
    dout = torch.randn(x.q.shape, generator=g, device=dev).to(torch.bfloat16)
    dq, dk, dv, dg = api.sparse_attn_bwd(cfg, x.q, x.k, x.v, x.gates, idx, dout, workspace=ws)
    torch.cuda.synchronize()
    del ws

    # invariants of dk, dv over the whole layer (fp64 sums on the GPU)
    s_dk = dk.double().sum(0)
    scale_k = dk.double().abs().sum(0)
    assert float((s_dk.abs() / scale_k.clamp_min(1e-30)).max()) <= 1e-3
    sg = torch.sigmoid(x.gates.double())
    want_v = ((sg[..., :1] + sg[..., 1:]) * dout.double()).sum(0)
    err_v = (dv.double().sum(0) - want_v).abs().max()
    assert float(err_v) <= 1e-3 * float(dv.double().abs().sum(0).max()), float(err_v)

    pb = O.Problem(L, H, 64, b, k, forced=forced, **geo)
    rng = np.random.default_rng(seed)
    blocks = sorted(set(rng.choice(cfg.nqb - 1, size=nsample - 1, replace=False).tolist())
                    | {cfg.nqb - 1})
    rows_t = torch.from_numpy(pb.rows_of(blocks)).to(dev)
    got_dq = dq.index_select(0, rows_t)
    got_dg = dg.index_select(0, rows_t)
    dout_rows = dout.index_select(0, rows_t).double().cpu().numpy()
    got_idx = np.ascontiguousarray(idx[:, blocks].cpu().numpy())
    heads = [0, H - 1]
    kblocks = sorted({0, pb.nb - 1} | set(rng.choice(pb.nb, size=2, replace=False).tolist()))
    key_rows = [pb.block_tokens(j) for j in kblocks]
    all_rows = torch.from_numpy(np.concatenate(key_rows)).to(dev)
    got_dk = dk.index_select(0, all_rows)[:, heads].cpu()
    got_dv = dv.index_select(0, all_rows)[:, heads].cpu()
    full_idx = idx.cpu().numpy() if name in BWD_KEYS else None
    full_dout = dout.double().cpu().numpy() if name in BWD_KEYS else None
    bits = [O.bf16_bits(t) for t in (x.q, x.k, x.v)]
    gates = x.gates.cpu().numpy()
    del x, dq, dk, dv, dg, dout
    torch.cuda.empty_cache()
    ref = O.backward(pb, *bits, gates, got_idx, dout_rows, qblocks=blocks)
    check_grad("dq", got_dq, ref.dq)
    check_grad("dgates", got_dg, ref.dgates)
    if name not in BWD_KEYS:
        return
    kc, vc = O.pool(pb, bits[1]), O.pool(pb, bits[2])
    for n_h, h in enumerate(heads):
        rk, rv = O.backward_keys(pb, *bits, gates, full_idx, full_dout, h, kblocks, kc=kc, vc=vc)
        want_k = np.concatenate([rk[a, :t.size] for a, t in enumerate(key_rows)])
        want_v = np.concatenate([rv[a, :t.size] for a, t in enumerate(key_rows)])
        check_grad(f"dk head {h}", got_dk[:, n_h], want_k)
        check_grad(f"dv head {h}", got_dv[:, n_h], want_v)
