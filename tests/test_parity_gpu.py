"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs, element by element, on small cases that span several
tiles with ragged tails, plus the edge cases of the method."""
import numpy as np
import pytest
import torch

import oracle
import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200.inputs import WORKLOADS, cu_seqlens, make_tensors, make_workload
from tests._util import (TOL, gpu_bwd, gpu_fwd, mask_kw, max_abs, oracle_bwd_slice,
                         oracle_fwd_slice, to_np)

pytestmark = pytest.mark.gpu

IMPLS = ["generic", "tensor_core"]


def small_case(B, T, H, D, NB, dtype=torch.bfloat16, Tk=None, seed=0, docs=None, q_off=0,
               k_off=0, causal=True):
    t = make_tensors(B, T, H, D, NB, dtype, Tk=Tk, seed=seed, device="cuda")
    t["scale"] = D ** -0.5
    t["cu_seqlens"] = None if docs is None else cu_seqlens(docs)
    t["max_seqlen"] = None if docs is None else max(docs)
    t["q_pos_offset"], t["k_pos_offset"], t["causal"] = q_off, k_off, causal
    return t


CASES = {
    "ragged_tiles_nb3": dict(B=2, T=300, H=2, D=128, NB=3),
    "d64_nb2": dict(B=1, T=517, H=2, D=64, NB=2),
    "varlen_nb4": dict(B=1, T=600, H=2, D=128, NB=4, docs=[1, 129, 0, 271, 199]),
    "frozen_target_offset": dict(B=1, T=130, H=2, D=128, NB=1, Tk=700, q_off=570),
    "noncausal_nb2": dict(B=1, T=200, H=2, D=128, NB=2, causal=False),
    "single_row_nb3": dict(B=1, T=1, H=3, D=128, NB=3),
    "masked_chunk_pair": dict(B=1, T=128, H=2, D=128, NB=1, q_off=0, k_off=256),
    "full_chunk_pair": dict(B=1, T=192, H=1, D=128, NB=1, Tk=256, q_off=1000, k_off=200),
    "varlen_chunk_pair": dict(B=1, T=160, H=2, D=64, NB=1, Tk=224, q_off=320, k_off=96,
                              docs=[150, 250, 300, 100]),
    # short documents: the two 128-row query tiles of a CTA see different key ranges
    "many_docs_nb2": dict(B=1, T=700, H=2, D=128, NB=2, docs=[5, 60, 3, 200, 90, 150, 80, 112]),
    # the last CTA's second query tile holds one row
    "second_tile_one_row": dict(B=1, T=385, H=2, D=64, NB=2),
}


def _run(case, impl):
    # every case is bf16 with D in {64, 128}, which the tensor-core path serves:
    # an EAGLE_ATTN_ERR_UNSUPPORTED here is a failure, not a skip
    c = dict(case)
    inp = small_case(c["B"], c["T"], c["H"], c["D"], c["NB"], Tk=c.get("Tk"), docs=c.get("docs"),
                     q_off=c.get("q_off", 0), k_off=c.get("k_off", 0),
                     causal=c.get("causal", True))
    out, lse = gpu_fwd(inp, impl=impl)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    return inp, out, lse


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name", list(CASES))
def test_fwd_matches_oracle(name, impl):
    inp, out, lse = _run(CASES[name], impl)
    tol = TOL[torch.bfloat16]
    kw = mask_kw(inp)
    B, H = inp["q"].shape[0], inp["q"].shape[2]
    for b in range(B):
        for h in range(H):
            ro, rl = oracle_fwd_slice(inp, b, h, **kw)
            assert max_abs(out[b:b + 1, :, h:h + 1], ro) <= tol["out"], (b, h)
            assert max_abs(lse[b:b + 1, h:h + 1], rl) <= tol["lse"], (b, h)


# (impl, deterministic): the CUDA-core backward, the tensor-core backward with
# five products per tile pair and fp32 atomics for dQ (the default), and the
# reproducible tensor-core pair (dK/dV kernel + dQ kernel)
BWD_MODES = [("generic", False), ("tensor_core", False), ("tensor_core", True)]


@pytest.mark.parametrize("impl,deterministic", BWD_MODES)
@pytest.mark.parametrize("name", ["ragged_tiles_nb3", "d64_nb2", "varlen_nb4",
                                  "frozen_target_offset", "noncausal_nb2", "single_row_nb3",
                                  "masked_chunk_pair", "varlen_chunk_pair", "many_docs_nb2",
                                  "full_chunk_pair"])
def test_bwd_matches_oracle(name, impl, deterministic):
    inp, out, lse = _run(CASES[name], impl)
    dq, dk, dv = gpu_bwd(inp, out, lse, impl=impl, deterministic=deterministic)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    tol = TOL[torch.bfloat16]
    kw = mask_kw(inp)
    B, H = inp["q"].shape[0], inp["q"].shape[2]
    for b in range(B):
        for h in range(H):
            rq, rk, rv = oracle_bwd_slice(inp, b, h, **kw)
            assert max_abs(dq[b:b + 1, :, h:h + 1], rq) <= tol["grad"], ("dq", b, h)
            assert max_abs(dk[b:b + 1, :, :, h:h + 1], rk) <= tol["grad"], ("dk", b, h)
            assert max_abs(dv[b:b + 1, :, :, h:h + 1], rv) <= tol["grad"], ("dv", b, h)


def test_tiny_fp32_config_fwd_bwd():
    """B=1 T=256 H=4 D=64 NB=2 fp32, scale 1/8: forward and backward within 1e-4."""
    w = WORKLOADS["tiny_fp32"]
    inp = make_workload(w, device="cuda")
    out, lse = gpu_fwd(inp)
    dq, dk, dv = gpu_bwd(inp, out, lse)
    torch.cuda.synchronize()
    ro, rl = oracle.fwd(to_np(inp["q"]), to_np(inp["cache_k"]), to_np(inp["cache_v"]), w.scale)
    rq, rk, rv = oracle.bwd(to_np(inp["q"]), to_np(inp["cache_k"]), to_np(inp["cache_v"]),
                            to_np(inp["grad_out"]), w.scale)
    tol = TOL[torch.float32]
    assert max_abs(out, ro) <= tol["out"]
    assert max_abs(lse, rl) <= tol["lse"]
    assert max_abs(dq, rq) <= tol["grad"]
    assert max_abs(dk, rk) <= tol["grad"]
    assert max_abs(dv, rv) <= tol["grad"]


@pytest.mark.parametrize("block_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128])
def test_merge_matches_oracle(block_dtype, D):
    g = torch.Generator().manual_seed(3)
    B, T, H = 2, 333, 3
    out = torch.randn(B, T, H, D, generator=g)
    lse = 3 * torch.randn(B, H, T, generator=g)
    bo = torch.randn(B, T, H, D, generator=g).to(block_dtype)
    bl = 3 * torch.randn(B, H, T, generator=g)
    lse[0, 0, :7] = -float("inf")          # empty running state
    out[0, :7, 0] = 0
    bl[0, 0, 3:11] = -float("inf")          # empty block (rows 3..6: both empty)
    bo[0, 3:11, 0] = 0
    eo, el = oracle.merge(out.double().numpy(), lse.double().numpy(), bo.double().numpy(),
                          bl.double().numpy())
    go, gl = out.cuda(), lse.cuda()
    ea.merge_out_lse(go, gl, bo.cuda(), bl.cuda())
    torch.cuda.synchronize()
    assert not torch.isnan(go).any() and not torch.isnan(gl).any()
    assert max_abs(go, eo) <= 1e-5
    assert max_abs(gl, el) <= 1e-5
    # init mode copies the block (_init_out_and_lse)
    ea.merge_out_lse(go, gl, bo.cuda(), bl.cuda(), init=True)
    torch.cuda.synchronize()
    assert max_abs(go, bo.float()) == 0 and max_abs(gl, bl) == 0


@pytest.mark.parametrize("D", [64, 128])
def test_merge_diag_matches_oracle(D):
    inp = small_case(1, 257, 2, D, 4, seed=5)
    blk0 = {**inp, "cache_k": inp["cache_k"][:, :1], "cache_v": inp["cache_v"][:, :1]}
    out, lse = gpu_fwd(blk0, out_dtype=torch.float32)
    ea.merge_diag(out, lse, inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"])
    torch.cuda.synchronize()
    for h in range(2):
        ro, rl = oracle_fwd_slice(inp, 0, h)
        assert max_abs(out[:, :, h:h + 1], ro) <= 2e-2
        assert max_abs(lse[:, h:h + 1], rl) <= 2e-3


@pytest.mark.parametrize("impl", IMPLS)
def test_zigzag_chunked_merge_equals_unchunked(impl):
    """Block 0 as 16 zig-zag chunks (emulated cp = 8): every (query chunk, key
    chunk) pair with its global offsets, merged with attn_merge_out_lse, then
    the diagonals with attn_merge_diag -- equal to the unchunked forward and to
    the oracle."""
    from online_softmax_merge_eagle_b200.schedules import zigzag_forward
    cp, c = 8, 80
    T, H, D, NB = 2 * cp * c, 2, 128, 4
    inp = small_case(1, T, H, D, NB, seed=6)
    ref_out, ref_lse = gpu_fwd(inp, impl=impl)
    got, got_lse = zigzag_forward(inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"], cp,
                                  impl=impl)
    torch.cuda.synchronize()
    assert max_abs(got, ref_out) <= 2e-2
    assert max_abs(got_lse, ref_lse) <= 2e-3
    for h in range(H):
        ro, rl = oracle_fwd_slice(inp, 0, h)
        assert max_abs(got[:, :, h:h + 1], ro) <= 2e-2
        assert max_abs(got_lse[:, h:h + 1], rl) <= 2e-3


def test_finalize_rounds_like_torch():
    x = torch.randn(3, 77, 5, 64, device="cuda")
    y = ea.finalize(x, torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y, x.to(torch.bfloat16))


def test_finalize_element_aligned_views():
    """Offsets that break 16-byte alignment (row ranges of an lse) take the
    element-wise path and give the same values."""
    x = torch.randn(1003, device="cuda")
    dst32 = torch.zeros(1003, device="cuda")
    dst16 = torch.zeros(1003, dtype=torch.bfloat16, device="cuda")
    ea.finalize(x[1:998], torch.float32, out=dst32[3:1000])
    ea.finalize(x[5:998], torch.bfloat16, out=dst16[1:994])
    torch.cuda.synchronize()
    assert torch.equal(dst32[3:1000], x[1:998])
    assert torch.equal(dst16[1:994], x[5:998].to(torch.bfloat16))


@pytest.mark.parametrize("impl", IMPLS)
def test_fwd_is_deterministic(impl):
    inp = small_case(1, 700, 2, 128, 3, seed=7)
    o1, l1 = gpu_fwd(inp, impl=impl)
    o2, l2 = gpu_fwd(inp, impl=impl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("impl", IMPLS)
def test_bwd_is_deterministic(impl):
    """deterministic = 1: no atomics in either backward, two runs agree bit for bit."""
    inp = small_case(1, 700, 2, 128, 3, seed=7)
    out, lse = gpu_fwd(inp)
    g1 = gpu_bwd(inp, out, lse, impl=impl, deterministic=True)
    g2 = gpu_bwd(inp, out, lse, impl=impl, deterministic=True)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_bwd_default_mode_repeats_within_rounding():
    """deterministic = 0 (the tensor-core default): dk and dv are still
    reproducible bit for bit (no atomics there); dq, summed with fp32 atomics,
    agrees between runs and with the reproducible pair to within bf16
    rounding."""
    inp = small_case(2, 900, 2, 128, 4, seed=9)
    out, lse = gpu_fwd(inp)
    a = gpu_bwd(inp, out, lse, impl="tensor_core")
    b = gpu_bwd(inp, out, lse, impl="tensor_core")
    c = gpu_bwd(inp, out, lse, impl="tensor_core", deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # one bf16 ulp at |x| < 4 is at most 2^-6
    assert all(max_abs(x, y) <= 2 ** -6 for x, y in zip(a, c))
    assert max_abs(a[0], b[0]) <= 2 ** -6


@pytest.mark.parametrize("Tq,Tk,NB", [(0, 0, 3), (0, 200, 1), (130, 0, 1)])
def test_empty_extents(Tq, Tk, NB):
    """Empty query or key ranges: no error; rows without keys get lse = -inf,
    out = 0 and dq = 0; keys without rows get dk = dv = 0."""
    t = make_tensors(1, Tq, 2, 128, NB, torch.bfloat16, Tk=Tk, seed=3, device="cuda")
    q, k, v, g = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    out, lse = ea.fwd(q, k, v)
    dq, dk, dv = ea.bwd(g, q, k, v, out, lse)
    torch.cuda.synchronize()
    assert ea.get_status() == 0
    assert out.shape == q.shape and lse.shape == (1, 2, Tq)
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    if Tq:
        assert torch.all(lse == -float("inf")) and torch.count_nonzero(out) == 0
        assert torch.count_nonzero(dq) == 0
    if Tk:
        assert torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0


def test_bad_cu_seqlens_sets_device_status_without_fault():
    inp = small_case(1, 64, 1, 128, 1, docs=[64])
    ea.clear_status()
    for bad, code in (([0, 40, 30, 64], 1), ([0, 64], 2), ([0, 32], 3)):
        inp["cu_seqlens"] = np.asarray(bad, dtype=np.int32)
        inp["max_seqlen"] = 10 if code == 2 else 64
        out, lse = gpu_fwd(inp, impl="generic")
        torch.cuda.synchronize()
        assert ea.get_status() == code
        ea.clear_status()
        assert ea.get_status() == 0
    # the context is still usable
    inp["cu_seqlens"] = np.asarray([0, 64], dtype=np.int32)
    inp["max_seqlen"] = 64
    out, lse = gpu_fwd(inp)
    torch.cuda.synchronize()
    assert ea.get_status() == 0 and torch.isfinite(lse).all()


def test_autograd_function_matches_explicit_calls():
    inp = small_case(1, 130, 2, 128, 2, seed=8)
    q = inp["q"].clone().requires_grad_()
    k = inp["cache_k"].clone().requires_grad_()
    v = inp["cache_v"].clone().requires_grad_()
    out = ea.eagle_attention(q, k, v, inp["scale"])
    out.backward(inp["grad_out"])
    o2, l2 = gpu_fwd(inp)
    dq, dk, dv = gpu_bwd(inp, o2, l2)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), o2)
    # the same library calls; dq may differ in its last bits (fp32 atomics)
    assert max_abs(q.grad, dq) <= 2 ** -6
    assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)
