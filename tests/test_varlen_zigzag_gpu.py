"""Varlen zig-zag halves ("eagle.zigzag_ring_attention": varlen throughout;
get_half_index / get_half_lse take the front and back half of every
document): packed documents, each cut into 2*cp chunks with rank r owning
chunks r and 2*cp-1-r of every document.  Forward and backward must equal the
unchunked packed (cu_seqlens) path, and the fp64 oracle on small cases."""
import numpy as np
import pytest
import torch

import oracle
import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200.inputs import WORKLOADS, cu_seqlens, make_tensors, make_workload
from online_softmax_merge_eagle_b200.schedules import varlen_zigzag_backward, varlen_zigzag_forward
from tests._util import TOL, max_abs

pytestmark = pytest.mark.gpu

TB = TOL[torch.bfloat16]


def _np(t):
    return t.detach().double().cpu().numpy()


@pytest.mark.parametrize("docs,H,D,NB,cp", [
    ([256, 64, 520, 184], 2, 128, 3, 4),
    ([48, 192, 12, 132], 2, 64, 2, 3),
])
def test_varlen_zigzag_matches_packed_and_oracle(docs, H, D, NB, cp):
    T = sum(docs)
    t = make_tensors(1, T, H, D, NB, torch.bfloat16, seed=7, device="cuda")
    q, k, v, g = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    scale = D ** -0.5
    cu_h = cu_seqlens(docs)
    cu_d = torch.as_tensor(cu_h, device="cuda")
    out, lse = varlen_zigzag_forward(q, k, v, scale, cu_h, cp=cp)
    dq, dk, dv = varlen_zigzag_backward(g, q, k, v, out, lse, scale, cu_h, cp=cp)
    ro, rl = ea.fwd(q, k, v, scale, cu_seqlens=cu_d, max_seqlen=max(docs))
    rq, rk, rv = ea.bwd(g, q, k, v, ro, rl, scale, cu_seqlens=cu_d, max_seqlen=max(docs))
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    assert max_abs(out, _np(ro)) <= TB["out"]
    assert max_abs(lse, _np(rl)) <= TB["lse"]
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert max_abs(a, _np(b)) <= TB["grad"]
    for h in (0, H - 1):
        qh, kh, vh, gh = (_np(q[:, :, h:h + 1]), _np(k[:, :, :, h:h + 1]),
                          _np(v[:, :, :, h:h + 1]), _np(g[:, :, h:h + 1]))
        oo, ol = oracle.fwd(qh, kh, vh, scale, cu_seqlens=np.asarray(cu_h))
        oq, ok_, ov = oracle.bwd(qh, kh, vh, gh, scale, cu_seqlens=np.asarray(cu_h))
        assert max_abs(out[:, :, h:h + 1], oo) <= TB["out"]
        assert max_abs(lse[:, h:h + 1], ol) <= TB["lse"]
        assert max_abs(dq[:, :, h:h + 1], oq) <= TB["grad"]
        assert max_abs(dk[:, :, :, h:h + 1], ok_) <= TB["grad"]
        assert max_abs(dv[:, :, :, h:h + 1], ov) <= TB["grad"]


@pytest.mark.parametrize("docs,H,D,NB,cp", [
    ([256, 64, 520, 184], 2, 128, 3, 4),
    ([48, 192, 12, 132], 2, 64, 2, 3),
])
def test_varlen_zigzag_single_launch_matches_packed_and_oracle(docs, H, D, NB, cp):
    """One launch per emulated rank (forward and backward) over its front and
    back chunk of every document: the packed path and the oracle."""
    T = sum(docs)
    t = make_tensors(1, T, H, D, NB, torch.bfloat16, seed=8, device="cuda")
    q, k, v, g = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    scale = D ** -0.5
    cu_h = cu_seqlens(docs)
    cu_d = torch.as_tensor(cu_h, device="cuda")
    out, lse = varlen_zigzag_forward(q, k, v, scale, cu_h, cp=cp, single_launch=True)
    dq, dk, dv = varlen_zigzag_backward(g, q, k, v, out, lse, scale, cu_h, cp=cp,
                                        single_launch=True)
    ro, rl = ea.fwd(q, k, v, scale, cu_seqlens=cu_d, max_seqlen=max(docs))
    rq, rk, rv = ea.bwd(g, q, k, v, ro, rl, scale, cu_seqlens=cu_d, max_seqlen=max(docs))
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    assert max_abs(out, _np(ro)) <= TB["out"]
    assert max_abs(lse, _np(rl)) <= TB["lse"]
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert max_abs(a, _np(b)) <= TB["grad"]
    for h in (0, H - 1):
        qh, kh, vh, gh = (_np(q[:, :, h:h + 1]), _np(k[:, :, :, h:h + 1]),
                          _np(v[:, :, :, h:h + 1]), _np(g[:, :, h:h + 1]))
        oo, ol = oracle.fwd(qh, kh, vh, scale, cu_seqlens=np.asarray(cu_h))
        oq, ok_, ov = oracle.bwd(qh, kh, vh, gh, scale, cu_seqlens=np.asarray(cu_h))
        assert max_abs(out[:, :, h:h + 1], oo) <= TB["out"]
        assert max_abs(lse[:, h:h + 1], ol) <= TB["lse"]
        assert max_abs(dq[:, :, h:h + 1], oq) <= TB["grad"]
        assert max_abs(dk[:, :, :, h:h + 1], ok_) <= TB["grad"]
        assert max_abs(dv[:, :, :, h:h + 1], ov) <= TB["grad"]


def test_varlen_zigzag_rejects_indivisible_documents():
    t = make_tensors(1, 100, 1, 64, 1, torch.bfloat16, grad=False, device="cuda")
    with pytest.raises(ValueError):
        varlen_zigzag_forward(t["q"], t["cache_k"], t["cache_v"], 0.125, [0, 30, 100], cp=2)


@pytest.mark.slow
@pytest.mark.parametrize("single", [False, True])
def test_varlen_zigzag_fullsize_equals_packed(single):
    """The varlen_zigzag_bf16 workload (T 32768, H 32, NB 4, 11 documents,
    16 chunks each): forward and backward equal the unchunked packed path."""
    w = WORKLOADS["varlen_zigzag_bf16"]
    cpu = make_workload(w)
    q, k, v, g = (cpu[n].cuda() for n in ("q", "cache_k", "cache_v", "grad_out"))
    cu_h = cpu["cu_seqlens"]
    cu_d = torch.as_tensor(cu_h, device="cuda")
    out, lse = varlen_zigzag_forward(q, k, v, w.scale, cu_h, cp=w.chunks // 2,
                                     single_launch=single)
    dq, dk, dv = varlen_zigzag_backward(g, q, k, v, out, lse, w.scale, cu_h, cp=w.chunks // 2,
                                        single_launch=single)
    ro, rl = ea.fwd(q, k, v, w.scale, cu_seqlens=cu_d, max_seqlen=cpu["max_seqlen"])
    rq, rk, rv = ea.bwd(g, q, k, v, ro, rl, w.scale, cu_seqlens=cu_d,
                        max_seqlen=cpu["max_seqlen"])
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    assert (out.float() - ro.float()).abs().max().item() <= TB["out"]
    assert (lse - rl).abs().max().item() <= TB["lse"]
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert (a.float() - b.float()).abs().max().item() <= TB["grad"]
    # documents never see each other, so a whole document is a problem of its
    # own: the oracle checks every row and key of the two shortest documents
    # and of the first one (chunk edges included), for two heads
    lens = np.diff(np.asarray(cu_h))
    pick = sorted(set(np.argsort(lens)[:2].tolist() + [0]))
    for d in pick:
        a, b = int(cu_h[d]), int(cu_h[d + 1])
        for h in (0, w.H - 1):
            qh = _np(cpu["q"][:, a:b, h:h + 1])
            kh = _np(cpu["cache_k"][:, :, a:b, h:h + 1])
            vh = _np(cpu["cache_v"][:, :, a:b, h:h + 1])
            gh = _np(cpu["grad_out"][:, a:b, h:h + 1])
            oo, ol = oracle.fwd(qh, kh, vh, w.scale)
            oq, ok_, ov = oracle.bwd(qh, kh, vh, gh, w.scale)
            assert max_abs(out[:, a:b, h:h + 1], oo) <= TB["out"], (d, h)
            assert max_abs(lse[:, h:h + 1, a:b], ol) <= TB["lse"], (d, h)
            assert max_abs(dq[:, a:b, h:h + 1], oq) <= TB["grad"], (d, h)
            assert max_abs(dk[:, :, a:b, h:h + 1], ok_) <= TB["grad"], (d, h)
            assert max_abs(dv[:, :, a:b, h:h + 1], ov) <= TB["grad"], (d, h)
