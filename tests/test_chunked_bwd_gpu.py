"""Chunked backward: the zig-zag schedule's per-(query chunk, key chunk)
backward against the final merged out / lse ("eagle.zigzag_ring_attention",
zigzag_ring_flash_attn_varlen_backward; "eagle.ulysses_attention",
_block0_backward), gradients summed in fp32 through
EAGLE_ATTN_GRAD_ACCUMULATE_F32.  It must equal the unchunked backward, and
the fp64 oracle on small cases."""
import numpy as np
import pytest
import torch

import oracle
import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200.inputs import make_tensors
from online_softmax_merge_eagle_b200.schedules import zigzag_backward, zigzag_forward
from tests._util import TOL, max_abs

pytestmark = pytest.mark.gpu

TB = TOL[torch.bfloat16]


def _inputs(T, H, D, NB, seed=3):
    t = make_tensors(1, T, H, D, NB, torch.bfloat16, seed=seed, device="cuda")
    return t["q"], t["cache_k"], t["cache_v"], t["grad_out"]


@pytest.mark.parametrize("single", [False, True])
@pytest.mark.parametrize("T,H,D,NB,cp", [(1024, 2, 128, 3, 2), (768, 2, 64, 2, 3),
                                         (1200, 2, 128, 2, 3)])
def test_chunked_bwd_matches_oracle_and_unchunked(T, H, D, NB, cp, single):
    """Per (query chunk, key chunk) pair, or (``single``) one launch per
    emulated rank over its two chunks (1200 rows, cp 3: chunks of 200 rows,
    not tile aligned)."""
    q, k, v, g = _inputs(T, H, D, NB)
    scale = D ** -0.5
    out, lse = zigzag_forward(q, k, v, scale, cp=cp, single_launch=single and T % 256 == 0)
    dq, dk, dv = zigzag_backward(g, q, k, v, out, lse, scale, cp=cp, single_launch=single)
    rq, rk, rv = ea.bwd(g, q, k, v, out, lse, scale)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    assert max_abs(dq, rq.double().cpu().numpy()) <= TB["grad"]
    assert max_abs(dk, rk.double().cpu().numpy()) <= TB["grad"]
    assert max_abs(dv, rv.double().cpu().numpy()) <= TB["grad"]
    for h in (0, H - 1):
        sl = lambda x: x.detach().double().cpu().numpy()  # noqa: E731
        oq, ok_, ov = oracle.bwd(sl(q[:, :, h:h + 1]), sl(k[:, :, :, h:h + 1]),
                                 sl(v[:, :, :, h:h + 1]), sl(g[:, :, h:h + 1]), scale)
        assert max_abs(dq[:, :, h:h + 1], oq) <= TB["grad"]
        assert max_abs(dk[:, :, :, h:h + 1], ok_) <= TB["grad"]
        assert max_abs(dv[:, :, :, h:h + 1], ov) <= TB["grad"]


@pytest.mark.parametrize("deterministic", [True, False])
def test_grad_accumulate_adds_exactly(deterministic):
    """Accumulating twice into zeros gives twice one accumulation, and one
    accumulation rounds to the stored (bf16) gradient: exactly with the
    reproducible backward; with the default one, dk / dv exactly and dq (its
    key tiles' contributions summed by fp32 atomics in varying order) to
    within fp32 rounding and one bf16 ulp."""
    q, k, v, g = _inputs(640, 2, 128, 3, seed=5)
    out, lse = ea.fwd(q, k, v)
    bufs = [torch.zeros(q.shape, dtype=torch.float32, device="cuda"),
            torch.zeros(k.shape, dtype=torch.float32, device="cuda"),
            torch.zeros(k.shape, dtype=torch.float32, device="cuda")]
    kw = dict(deterministic=deterministic)
    ea.bwd(g, q, k, v, out, lse, dq=bufs[0], dk=bufs[1], dv=bufs[2], grad_accumulate=True, **kw)
    once = [b.clone() for b in bufs]
    ea.bwd(g, q, k, v, out, lse, dq=bufs[0], dk=bufs[1], dv=bufs[2], grad_accumulate=True, **kw)
    ref = ea.bwd(g, q, k, v, out, lse, **kw)
    torch.cuda.synchronize()
    for i, (b, o, r) in enumerate(zip(bufs, once, ref)):
        if deterministic or i > 0:
            assert torch.equal(b, 2 * o)
            assert torch.equal(o.to(torch.bfloat16), r)
        else:
            assert max_abs(b, 2 * o) <= 1e-5
            assert max_abs(o.to(torch.bfloat16), r) <= 2 ** -6


@pytest.mark.slow
@pytest.mark.parametrize("single", [False, True])
def test_chunked_bwd_fullsize_equals_unchunked(single):
    """131072 positions, 16 zig-zag chunks (emulated cp = 8), NB = 4, H = 8:
    every gradient of the chunked backward (per pair, or one launch per rank)
    equals the unchunked one."""
    q, k, v, g = _inputs(131072, 8, 128, 4, seed=0)
    scale = 128 ** -0.5
    out, lse = zigzag_forward(q, k, v, scale, cp=8, single_launch=single)
    dq, dk, dv = zigzag_backward(g, q, k, v, out, lse, scale, cp=8, single_launch=single)
    rq, rk, rv = ea.bwd(g, q, k, v, out, lse, scale)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        assert (a.float() - b.float()).abs().max().item() <= TB["grad"]
    # the oracle on the causal prefix of two chunks (rows 0 .. 16383, across the
    # first chunk edge), two heads: a row's dq and its diagonal blocks' dk / dv
    # depend only on keys at or before it, so the prefix problem gives them
    # exactly (block-0 dk / dv of a key need every later row: checked above
    # against the unchunked path, which the full-size slice tests pin)
    n = 2 * (131072 // 16)
    sl = lambda x: x.detach().double().cpu().numpy()  # noqa: E731
    for h in (0, 7):
        oq, ok_, ov = oracle.bwd(sl(q[:, :n, h:h + 1]), sl(k[:, :, :n, h:h + 1]),
                                 sl(v[:, :, :n, h:h + 1]), sl(g[:, :n, h:h + 1]), scale)
        assert max_abs(dq[:, :n, h:h + 1], oq) <= TB["grad"], h
        assert max_abs(rq[:, :n, h:h + 1], oq) <= TB["grad"], h  # the unchunked path too
        assert max_abs(dk[:, 1:, :n, h:h + 1], ok_[:, 1:]) <= TB["grad"], h
        assert max_abs(dv[:, 1:, :n, h:h + 1], ov[:, 1:]) <= TB["grad"], h
