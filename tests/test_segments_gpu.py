"""Query segments (ABI 4: q_tiles with q_tile_rows): lists of row ranges of at
most 128 rows, not aligned to tiles, so that one launch serves an emulated
rank's front and back half of every document ("eagle.zigzag_ring_attention",
get_half_index, and zigzag_ring_flash_attn_varlen_backward for the backward).

The forward over a segment list computes exactly those rows.  The backward over
a sorted, disjoint list is the gradient through exactly those rows' outputs:
the same as the whole backward with grad_out zero on every other row (their
dq untouched), which is what the oracle checks."""
import numpy as np
import pytest
import torch

import oracle
import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200.inputs import cu_seqlens, make_tensors
from tests._util import TOL, max_abs

pytestmark = pytest.mark.gpu

TB = TOL[torch.bfloat16]


def _np(t):
    return t.detach().double().cpu().numpy()


def _case(T, H, D, NB, seed, docs=None):
    t = make_tensors(1, T, H, D, NB, torch.bfloat16, seed=seed, device="cuda")
    kw = {}
    if docs is not None:
        kw = dict(cu_seqlens=torch.as_tensor(cu_seqlens(docs), device="cuda"),
                  max_seqlen=max(docs))
    return t, kw


# row ranges: ragged, unaligned, crossing 128-row tile and document edges
RANGES = {
    "dense_d128": dict(T=700, H=2, D=128, NB=3, docs=None,
                       ranges=[(3, 40), (130, 390), (455, 456), (512, 700)]),
    "varlen_d64": dict(T=600, H=2, D=64, NB=2, docs=[1, 129, 0, 271, 199],
                       ranges=[(0, 77), (120, 131), (200, 333), (400, 600)]),
}


@pytest.mark.parametrize("name", list(RANGES))
def test_forward_over_segments(name):
    c = RANGES[name]
    t, kw = _case(c["T"], c["H"], c["D"], c["NB"], seed=31, docs=c["docs"])
    tiles, rows = ea.query_segments(c["ranges"], "cuda")
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full((1, c["H"], c["T"]), 7.0, device="cuda")
    ea.fwd(t["q"], t["cache_k"], t["cache_v"], out=out, lse=lse, q_tiles=tiles, q_tile_rows=rows,
           **kw)
    ro, rl = ea.fwd(t["q"], t["cache_k"], t["cache_v"], **kw)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    own = torch.zeros(c["T"], dtype=torch.bool)
    for a, b in c["ranges"]:
        own[a:b] = True
    own = own.cuda()
    assert max_abs(out[:, own], _np(ro[:, own])) <= TB["out"]
    assert max_abs(lse[:, :, own], _np(rl[:, :, own])) <= TB["lse"]
    assert torch.isnan(out[:, ~own].float()).all() and (lse[:, :, ~own] == 7.0).all()
    cu = None if c["docs"] is None else np.asarray(cu_seqlens(c["docs"]))
    for h in range(c["H"]):
        oo, ol = oracle.fwd(_np(t["q"][:, :, h:h + 1]), _np(t["cache_k"][:, :, :, h:h + 1]),
                            _np(t["cache_v"][:, :, :, h:h + 1]), c["D"] ** -0.5, cu_seqlens=cu)
        own_np = own.cpu().numpy()
        assert max_abs(out[:, own, h:h + 1], oo[:, own_np]) <= TB["out"]
        assert max_abs(lse[:, h:h + 1, own], ol[:, :, own_np]) <= TB["lse"]


@pytest.mark.parametrize("accumulate", [False, True])
@pytest.mark.parametrize("name", list(RANGES))
def test_backward_over_segments_is_the_masked_gradient(name, accumulate):
    c = RANGES[name]
    t, kw = _case(c["T"], c["H"], c["D"], c["NB"], seed=32, docs=c["docs"])
    q, k, v, g = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    out, lse = ea.fwd(q, k, v, **kw)
    own = torch.zeros(c["T"], dtype=torch.bool)
    for a, b in c["ranges"]:
        own[a:b] = True
    own = own.cuda()
    g_masked = g.clone()
    g_masked[:, ~own] = 0
    tiles, rows = ea.query_segments(c["ranges"], "cuda")
    if accumulate:
        bufs = [torch.zeros(x.shape, dtype=torch.float32, device="cuda") for x in (q, k, v)]
        dq, dk, dv = ea.bwd(g, q, k, v, out, lse, dq=bufs[0], dk=bufs[1], dv=bufs[2],
                            grad_accumulate=True, q_tiles=tiles, q_tile_rows=rows, **kw)
    else:
        dq = torch.full_like(q, float("nan"))
        dk = torch.full_like(k, float("nan"))
        dv = torch.full_like(v, float("nan"))
        ea.bwd(g, q, k, v, out, lse, dq=dq, dk=dk, dv=dv, q_tiles=tiles, q_tile_rows=rows, **kw)
    rq, rk, rv = ea.bwd(g_masked, q, k, v, out, lse, **kw)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    # dq and the diagonal blocks: the listed rows; block 0 of dk / dv: every key
    assert max_abs(dq[:, own], _np(rq[:, own])) <= TB["grad"]
    assert max_abs(dk[:, 1:, own], _np(rk[:, 1:, own])) <= TB["grad"]
    assert max_abs(dv[:, 1:, own], _np(rv[:, 1:, own])) <= TB["grad"]
    assert max_abs(dk[:, :1], _np(rk[:, :1])) <= TB["grad"]
    assert max_abs(dv[:, :1], _np(rv[:, :1])) <= TB["grad"]
    if not accumulate:  # the other rows untouched
        assert torch.isnan(dq[:, ~own].float()).all()
        assert torch.isnan(dk[:, 1:, ~own].float()).all()
    else:
        assert (dq[:, ~own] == 0).all() and (dk[:, 1:, ~own] == 0).all()
    cu = None if c["docs"] is None else np.asarray(cu_seqlens(c["docs"]))
    own_np = own.cpu().numpy()
    for h in range(c["H"]):
        oq, ok_, ov = oracle.bwd(_np(q[:, :, h:h + 1]), _np(k[:, :, :, h:h + 1]),
                                 _np(v[:, :, :, h:h + 1]), _np(g_masked[:, :, h:h + 1]),
                                 c["D"] ** -0.5, cu_seqlens=cu)
        assert max_abs(dq[:, own, h:h + 1], oq[:, own_np]) <= TB["grad"]
        assert max_abs(dk[:, :1, :, h:h + 1], ok_[:, :1]) <= TB["grad"]
        assert max_abs(dv[:, :1, :, h:h + 1], ov[:, :1]) <= TB["grad"]
        assert max_abs(dk[:, 1:, own, h:h + 1], ok_[:, 1:, own_np]) <= TB["grad"]


def test_segment_lists_out_of_range_or_order_raise_device_status():
    """Entries out of range (forward) and a list out of order (backward) set
    EAGLE_ATTN_DEV_BAD_TILE; the kernels skip those entries, and the context
    stays usable."""
    t, _ = _case(512, 1, 128, 1, seed=33)
    q, k, v, g = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    i32 = dict(dtype=torch.int32, device="cuda")
    ea.clear_status()
    ea.fwd(q, k, v, q_tiles=torch.tensor([0, 500], **i32),
           q_tile_rows=torch.tensor([129, 20], **i32))  # 129 rows; 500 + 20 past Tq
    torch.cuda.synchronize()
    assert ea.get_status() == 5
    ea.clear_status()
    out, lse = ea.fwd(q, k, v)
    ea.bwd(g, q, k, v, out, lse, q_tiles=torch.tensor([200, 100], **i32),
           q_tile_rows=torch.tensor([50, 50], **i32))  # out of order
    torch.cuda.synchronize()
    assert ea.get_status() == 5
    ea.clear_status()
    ro, rl = ea.fwd(q, k, v)
    torch.cuda.synchronize()
    assert ea.get_status() == 0 and torch.equal(ro, out)
