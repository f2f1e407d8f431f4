"""Helpers shared by the GPU parity tests (no attention arithmetic here: the
expected values come from the oracle package)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import online_softmax_merge_eagle_b200 as ea

# Tolerances (max-abs), from the stated targets: bf16 inputs with fp32
# accumulation: out/dq/dk/dv 2e-2, lse 2e-3; fp32 inputs: 1e-4.
TOL = {
    torch.bfloat16: dict(out=2e-2, lse=2e-3, grad=2e-2),
    torch.float32: dict(out=1e-4, lse=1e-4, grad=1e-4),
}


def max_abs(a, b) -> float:
    a = a.detach().double().cpu().numpy() if isinstance(a, torch.Tensor) else np.asarray(a)
    b = b.detach().double().cpu().numpy() if isinstance(b, torch.Tensor) else np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        d = np.where(both_inf, 0.0, np.abs(a - b))
    if d.size == 0:
        return 0.0
    return float(np.nanmax(np.where(np.isnan(d), np.inf, d)))


def to_np(t):
    return t.detach().to("cpu").double().numpy()


def slice_bh(t, b, h, kind):
    """(b, h) slice of a q-like [B,T,H,D] or cache-like [B,NB,T,H,D] tensor,
    kept 4-D / 5-D with B = H = 1, as fp64 numpy."""
    if kind == "q":
        return to_np(t[b:b + 1, :, h:h + 1, :])
    return to_np(t[b:b + 1, :, :, h:h + 1, :])


def oracle_fwd_slice(inp, b, h, rows=None, **mask):
    q = slice_bh(inp["q"], b, h, "q")
    k = slice_bh(inp["cache_k"], b, h, "kv")
    v = slice_bh(inp["cache_v"], b, h, "kv")
    return oracle.fwd(q, k, v, inp["scale"], rows=rows, **mask)


def oracle_bwd_slice(inp, b, h, **mask):
    q = slice_bh(inp["q"], b, h, "q")
    k = slice_bh(inp["cache_k"], b, h, "kv")
    v = slice_bh(inp["cache_v"], b, h, "kv")
    g = slice_bh(inp["grad_out"], b, h, "q")
    return oracle.bwd(q, k, v, g, inp["scale"], **mask)


def mask_kw(inp):
    kw = {}
    if inp.get("cu_seqlens") is not None:
        kw["cu_seqlens"] = np.asarray(inp["cu_seqlens"])
    kw["q_pos_offset"] = inp.get("q_pos_offset", 0)
    kw["k_pos_offset"] = inp.get("k_pos_offset", 0)
    kw["causal"] = inp.get("causal", True)
    return kw


def gpu_fwd(inp, impl="auto", out_dtype=None):
    return ea.fwd(inp["q"], inp["cache_k"], inp["cache_v"], inp["scale"],
                  cu_seqlens=inp.get("cu_seqlens"), max_seqlen=inp.get("max_seqlen"),
                  q_pos_offset=inp.get("q_pos_offset", 0), k_pos_offset=inp.get("k_pos_offset", 0),
                  causal=inp.get("causal", True), impl=impl, out_dtype=out_dtype)


def gpu_bwd(inp, out, lse, impl="auto", deterministic=False):
    return ea.bwd(inp["grad_out"], inp["q"], inp["cache_k"], inp["cache_v"], out, lse,
                  inp["scale"], cu_seqlens=inp.get("cu_seqlens"), max_seqlen=inp.get("max_seqlen"),
                  q_pos_offset=inp.get("q_pos_offset", 0), k_pos_offset=inp.get("k_pos_offset", 0),
                  causal=inp.get("causal", True), impl=impl, deterministic=deterministic)
