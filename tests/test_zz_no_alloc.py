"""eagle_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (a plugin inside a framework that owns all device memory and offers no
workspace hook, or a loop that must not call cudaMalloc because it can
synchronise the device).  Its scratch is a fixed 32 MiB array inside the
library, shared by every call, so the test calls it twice in a row and checks
both results against eagle_attn_bwd with a caller-provided workspace.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process (its first call on the device performs the scratch set-up)."""
import ctypes

import pytest
import torch

import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200 import _lib
from online_softmax_merge_eagle_b200.inputs import make_tensors
from tests._util import TOL, max_abs


def _params(inp, out, lse, dq, dk, dv, impl="auto"):
    p, _ = ea._params(inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"], None, None, 0, 0,
                      True, impl)
    p.out_dtype = _lib.BF16
    p.out, p.lse, p.grad_out = out.data_ptr(), lse.data_ptr(), inp["grad_out"].data_ptr()
    p.dq, p.dk, p.dv = dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    p.workspace, p.workspace_bytes = None, 0
    return p


@pytest.mark.gpu
@pytest.mark.parametrize("impl", ["auto", "generic"])
def test_bwd_noalloc_matches_bwd_on_two_calls_in_a_row(impl):
    inp = make_tensors(1, 300, 2, 128, 3, torch.bfloat16, seed=11, device="cuda")
    inp["scale"] = 128 ** -0.5
    out, lse = ea.fwd(inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"])
    ref = ea.bwd(inp["grad_out"], inp["q"], inp["cache_k"], inp["cache_v"], out, lse,
                 inp["scale"], impl=impl)
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    tol = TOL[torch.bfloat16]["grad"]
    for _ in range(2):
        dq = torch.full_like(inp["q"], float("nan"))
        dk = torch.full_like(inp["cache_k"], float("nan"))
        dv = torch.full_like(inp["cache_v"], float("nan"))
        p = _params(inp, out, lse, dq, dk, dv, impl)
        rc = lib.eagle_attn_bwd_noalloc(ctypes.byref(p), stream)
        assert rc == 0, _lib.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert ea.get_status() == 0
        for got, want in zip((dq, dk, dv), ref):
            assert not torch.isnan(got).any()
            assert max_abs(got, want) <= tol


@pytest.mark.gpu
def test_bwd_noalloc_after_leftovers_of_larger_and_other_calls():
    """The scratch keeps whatever the last call left there.  Fill it with a
    larger problem's data, then with a CUDA-core call's, and run smaller
    problems through eagle_attn_bwd_noalloc: each still matches eagle_attn_bwd
    (the call clears what must start at zero itself)."""
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    tol = TOL[torch.bfloat16]["grad"]

    def case(T, H, NB, seed, impl):
        inp = make_tensors(1, T, H, 128, NB, torch.bfloat16, seed=seed, device="cuda")
        inp["scale"] = 128 ** -0.5
        out, lse = ea.fwd(inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"])
        dq, dk, dv = (torch.full_like(x, float("nan"))
                      for x in (inp["q"], inp["cache_k"], inp["cache_v"]))
        p = _params(inp, out, lse, dq, dk, dv, impl)
        rc = lib.eagle_attn_bwd_noalloc(ctypes.byref(p), stream)
        assert rc == 0, _lib.STATUS.get(rc, rc)
        ref = ea.bwd(inp["grad_out"], inp["q"], inp["cache_k"], inp["cache_v"], out, lse,
                     inp["scale"], impl=impl)
        torch.cuda.synchronize()
        assert ea.get_status() == 0
        for got, want in zip((dq, dk, dv), ref):
            assert not torch.isnan(got).any()
            assert max_abs(got, want) <= tol

    case(2048, 8, 4, 21, "auto")     # the larger problem: scratch full of its sums
    case(300, 2, 1, 22, "auto")      # smaller, no diagonal blocks
    case(400, 2, 3, 23, "generic")   # the CUDA-core path's use of the scratch
    case(260, 3, 2, 24, "auto")


def test_bwd_noalloc_ignores_the_workspace_fields():
    """Host-side: a stale, misaligned p->workspace does not make the call fail
    its argument checks (the fields are documented as ignored); the call gets
    as far as the scratch-size check."""
    lib = _lib.load()
    p = _lib.Params()
    lib.eagle_attn_params_init(ctypes.byref(p))
    p.B, p.Tq, p.Tk, p.H, p.D, p.num_blocks = 1, 8192, 8192, 16, 128, 2
    p.scale = 128 ** -0.5
    fake = 1 << 20
    p.q = p.cache_k = p.cache_v = p.out = p.lse = fake
    p.grad_out = p.dq = p.dk = p.dv = fake
    p.workspace, p.workspace_bytes = fake + 3, 7
    rc = lib.eagle_attn_bwd_noalloc(ctypes.byref(p), None)
    assert _lib.STATUS[rc] == "EAGLE_ATTN_ERR_SCRATCH_LIMIT"


def test_bwd_noalloc_rejects_problems_beyond_its_scratch():
    """Host-side check, before any CUDA call: B*Tq*H*(4D + 4) bytes of scratch
    above 32 MiB is refused with EAGLE_ATTN_ERR_SCRATCH_LIMIT."""
    lib = _lib.load()
    p = _lib.Params()
    lib.eagle_attn_params_init(ctypes.byref(p))
    p.B, p.Tq, p.Tk, p.H, p.D, p.num_blocks = 1, 8192, 8192, 16, 128, 2
    p.scale = 128 ** -0.5
    fake = 1 << 20  # aligned and never dereferenced: the size check comes first
    p.q = p.cache_k = p.cache_v = p.out = p.lse = fake
    p.grad_out = p.dq = p.dk = p.dv = fake
    need = lib.eagle_attn_bwd_workspace_size(ctypes.byref(p))
    assert need > _lib.NOALLOC_SCRATCH_BYTES
    rc = lib.eagle_attn_bwd_noalloc(ctypes.byref(p), None)
    assert _lib.STATUS[rc] == "EAGLE_ATTN_ERR_SCRATCH_LIMIT"
    assert "scratch" in lib.eagle_attn_strerror(rc).decode()
