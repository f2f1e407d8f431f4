"""EAGLE-3 mixed joint-softmax attention on B200 (sm_100a) -- Python binding.

A thin layer over the C ABI of libeagleattn (include/eagleattn.h): it reads
shapes and strides off torch tensors, allocates outputs with torch, and calls
the library on torch's current CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
calls fail loudly when the library is missing.

The method (NeMo AutoModel API page "eagle.ring_attention", class
_CachedRingAttention): block 0 is causal attention of q against the sequence
K/V cache_k[:, 0] / cache_v[:, 0] (optionally packed by cu_seqlens documents,
"eagle.ulysses_attention" _block0_forward), blocks i >= 1 are per-position
diagonals with logit (q_t . k_i_t) * scale and value v_i_t, all in one
softmax through the log-sum-exp merge.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import BF16, F32, GRAD_ACCUMULATE_F32, IMPL, Params

__all__ = [
    "EagleAttnError", "fwd", "bwd", "merge_out_lse", "merge_diag", "finalize", "get_status",
    "clear_status", "bwd_workspace_size", "eagle_attention", "library_path", "launch_count",
    "bwd_noalloc", "query_segments",
]

library_path = _lib.LIB_PATH


class EagleAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        lib = _lib.load()
        msg = lib.eagle_attn_strerror(code).decode()
        super().__init__(f"{what}: {_lib.STATUS.get(code, code)} ({msg})")
        self.code = code


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise EagleAttnError(rc, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _torch_dtype(code: int) -> torch.dtype:
    return torch.float32 if code == F32 else torch.bfloat16


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _cu_tensor(cu_seqlens, device):
    if cu_seqlens is None:
        return None
    if not isinstance(cu_seqlens, torch.Tensor):
        cu_seqlens = torch.as_tensor(cu_seqlens, dtype=torch.int32)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    return cu_seqlens.to(device)


def _params(q, cache_k, cache_v, scale, cu_seqlens, max_seqlen, q_pos_offset, k_pos_offset,
            causal, impl) -> tuple[Params, torch.Tensor | None]:
    if q.dim() != 4 or cache_k.dim() != 5 or cache_v.shape != cache_k.shape:
        raise ValueError("q must be [B,T,H,D] and cache_k/cache_v [B,NB,Tk,H,D]")
    if not (q.is_cuda and cache_k.is_cuda and cache_v.is_cuda):
        raise ValueError("tensors must be on a CUDA device")
    B, Tq, H, D = q.shape
    if cache_k.shape[0] != B or cache_k.shape[3] != H or cache_k.shape[4] != D:
        raise ValueError("cache_k shape does not match q")
    if cache_k.stride() != cache_v.stride() or cache_k.dtype != q.dtype or cache_v.dtype != q.dtype:
        raise ValueError("cache_k and cache_v must share dtype and strides with each other and q")
    for t in (q, cache_k):
        if t.stride(-1) != 1 or t.stride(-2) != D:
            raise ValueError("the head and feature dims must be dense ([.., H, D] contiguous)")
    p = Params()
    _lib.load().eagle_attn_params_init(ctypes.byref(p))
    p.dtype = _dt(q)
    p.out_dtype = p.dtype
    p.impl = IMPL[impl]
    p.B, p.Tq, p.H, p.D = B, Tq, H, D
    p.num_blocks, p.Tk = cache_k.shape[1], cache_k.shape[2]
    p.causal = 1 if causal else 0
    p.scale = float(D ** -0.5 if scale is None else scale)
    p.q_pos_offset, p.k_pos_offset = int(q_pos_offset), int(k_pos_offset)
    cu = _cu_tensor(cu_seqlens, q.device)
    if cu is not None:
        p.cu_seqlens = cu.data_ptr()
        p.num_docs = cu.numel() - 1
        p.max_seqlen = int(max_seqlen) if max_seqlen is not None else 0
    p.q_stride_b, p.q_stride_t = q.stride(0), q.stride(1)
    p.kv_stride_b, p.kv_stride_blk, p.kv_stride_t = cache_k.stride(0), cache_k.stride(1), cache_k.stride(2)
    p.q, p.cache_k, p.cache_v = q.data_ptr(), cache_k.data_ptr(), cache_v.data_ptr()
    return p, cu


def _same_layout(a, b) -> bool:
    """Equal shapes and equal strides on every dim of extent > 1."""
    return a.shape == b.shape and all(
        n == 1 or sa == sb for n, sa, sb in zip(a.shape, a.stride(), b.stride()))


def _like_q(q, dtype):
    return torch.empty_strided(q.shape, q.stride(), dtype=dtype, device=q.device)


def _prof(p, prof):
    if prof is not None:
        for e in prof:
            if not e.cuda_event:  # torch creates the CUDA event on first record
                e.record()
        p.prof_start, p.prof_stop = prof[0].cuda_event, prof[1].cuda_event


def _set_tiles(p, q_tiles, q_tile_rows):
    """q_tiles / q_tile_rows (int32 CUDA tensors of the same length) into *p."""
    if q_tiles is None:
        if q_tile_rows is not None:
            raise ValueError("q_tile_rows needs q_tiles")
        return
    for t in (q_tiles, q_tile_rows):
        if t is not None and (t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous()):
            raise ValueError("q_tiles / q_tile_rows must be contiguous int32 CUDA tensors")
    if q_tile_rows is not None and q_tile_rows.numel() != q_tiles.numel():
        raise ValueError("q_tile_rows needs one entry per q_tiles entry")
    p.q_tiles, p.num_q_tiles = q_tiles.data_ptr(), q_tiles.numel()
    if q_tile_rows is not None:
        p.q_tile_rows = q_tile_rows.data_ptr()


def query_segments(row_ranges, device) -> tuple[torch.Tensor, torch.Tensor]:
    """(q_tiles, q_tile_rows) for the union of half-open row ranges [a, b):
    sorted, disjoint segments of at most 128 rows (ranges must not overlap)."""
    starts, rows = [], []
    for a, b in sorted(row_ranges):
        for t in range(a, b, 128):
            starts.append(t)
            rows.append(min(128, b - t))
    return (torch.tensor(starts, dtype=torch.int32).to(device, non_blocking=True),
            torch.tensor(rows, dtype=torch.int32).to(device, non_blocking=True))


def fwd(q, cache_k, cache_v, scale=None, cu_seqlens=None, max_seqlen=None, q_pos_offset=0,
        k_pos_offset=0, causal=True, out_dtype=None, impl="auto", out=None, lse=None, prof=None,
        q_tiles=None, q_tile_rows=None):
    """Forward: returns (out [B,Tq,H,D], lse [B,H,Tq] fp32).  ``out_dtype``
    torch.float32 keeps the block unrounded for a later merge.  ``prof`` =
    (start, stop) torch.cuda.Event pair recorded around the main kernel.
    ``q_tiles``: int32 CUDA tensor of query row starts (multiples of 128); only
    those 128-row tiles are computed, the other rows of out / lse untouched.
    With ``q_tile_rows`` (rows per entry, 1..128) the starts need no alignment:
    segments of any length (``query_segments`` builds them from row ranges)."""
    p, cu = _params(q, cache_k, cache_v, scale, cu_seqlens, max_seqlen, q_pos_offset,
                    k_pos_offset, causal, impl)
    od = q.dtype if out_dtype is None else out_dtype
    p.out_dtype = _dt(torch.empty(0, dtype=od))
    if out is None:
        out = _like_q(q, od)
    if not _same_layout(out, q) or out.dtype != od:
        raise ValueError("out must have q's strides and out_dtype")
    if lse is None:
        lse = torch.empty((p.B, p.H, p.Tq), dtype=torch.float32, device=q.device)
    if not lse.is_contiguous() or lse.shape != (p.B, p.H, p.Tq):
        raise ValueError("lse must be a contiguous fp32 [B, H, Tq] tensor")
    p.out, p.lse = out.data_ptr(), lse.data_ptr()
    _set_tiles(p, q_tiles, q_tile_rows)
    _prof(p, prof)
    _check(_lib.load().eagle_attn_fwd(ctypes.byref(p), _stream()), "eagle_attn_fwd")
    return out, lse


def bwd_workspace_size(q, cache_k, cache_v, **kw) -> int:
    p, _ = _params(q, cache_k, cache_v, kw.get("scale"), kw.get("cu_seqlens"), kw.get("max_seqlen"),
                   kw.get("q_pos_offset", 0), kw.get("k_pos_offset", 0), kw.get("causal", True),
                   kw.get("impl", "auto"))
    return int(_lib.load().eagle_attn_bwd_workspace_size(ctypes.byref(p)))


def bwd(grad_out, q, cache_k, cache_v, out, lse, scale=None, cu_seqlens=None, max_seqlen=None,
        q_pos_offset=0, k_pos_offset=0, causal=True, deterministic=False, impl="auto",
        workspace=None, dq=None, dk=None, dv=None, prof=None, grad_accumulate=False,
        q_tiles=None, q_tile_rows=None):
    """Backward against the MERGED (out, lse): returns (dq, dk, dv) with dk/dv
    covering every block.  ``grad_accumulate``: dq/dk/dv are given fp32 buffers
    (q's / cache_k's element strides) and the call adds its gradient to them
    (EAGLE_ATTN_GRAD_ACCUMULATE_F32, the chunked schedule's mode).
    ``q_tiles`` / ``q_tile_rows``: sorted, disjoint query segments; only those
    rows' part of the gradient (their dq, their contributions to dk / dv)."""
    p, cu = _params(q, cache_k, cache_v, scale, cu_seqlens, max_seqlen, q_pos_offset,
                    k_pos_offset, causal, impl)
    if not _same_layout(grad_out, q) or not _same_layout(out, q):
        raise ValueError("grad_out and out must have q's strides")
    if grad_out.dtype != q.dtype:
        raise ValueError("grad_out must have q's dtype")
    p.out_dtype = _dt(out)
    p.deterministic = 1 if deterministic else 0
    if grad_accumulate:
        if dq is None or dk is None or dv is None:
            raise ValueError("grad_accumulate needs the fp32 dq, dk, dv buffers")
        if any(t.dtype != torch.float32 for t in (dq, dk, dv)):
            raise ValueError("grad_accumulate buffers must be fp32")
        if not _same_layout(dq, q) or not _same_layout(dk, cache_k) or not _same_layout(dv, cache_k):
            raise ValueError("dq must have q's strides and dk/dv cache_k's")
        p.grad_mode = GRAD_ACCUMULATE_F32
    if dq is None:
        dq = _like_q(q, q.dtype)
    if dk is None:
        dk = torch.empty_strided(cache_k.shape, cache_k.stride(), dtype=q.dtype, device=q.device)
    if dv is None:
        dv = torch.empty_strided(cache_k.shape, cache_k.stride(), dtype=q.dtype, device=q.device)
    p.out, p.lse, p.grad_out = out.data_ptr(), lse.data_ptr(), grad_out.data_ptr()
    p.dq, p.dk, p.dv = dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    _set_tiles(p, q_tiles, q_tile_rows)
    lib = _lib.load()
    need = int(lib.eagle_attn_bwd_workspace_size(ctypes.byref(p)))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = workspace.numel() * workspace.element_size()
    _prof(p, prof)
    _check(lib.eagle_attn_bwd(ctypes.byref(p), _stream()), "eagle_attn_bwd")
    return dq, dk, dv


def bwd_noalloc(grad_out, q, cache_k, cache_v, out, lse, dq, dk, dv, scale=None,
                cu_seqlens=None, max_seqlen=None, q_pos_offset=0, k_pos_offset=0, causal=True,
                impl="auto"):
    """eagle_attn_bwd_noalloc: the backward with the library's fixed scratch
    buffer instead of a caller workspace, for callers that cannot allocate
    device memory.  dq/dk/dv must be given (nothing is allocated here)."""
    p, cu = _params(q, cache_k, cache_v, scale, cu_seqlens, max_seqlen, q_pos_offset,
                    k_pos_offset, causal, impl)
    if not _same_layout(grad_out, q) or not _same_layout(out, q) or not _same_layout(dq, q):
        raise ValueError("grad_out, out and dq must have q's strides")
    if not _same_layout(dk, cache_k) or not _same_layout(dv, cache_k):
        raise ValueError("dk and dv must have cache_k's strides")
    p.out_dtype = _dt(out)
    p.out, p.lse, p.grad_out = out.data_ptr(), lse.data_ptr(), grad_out.data_ptr()
    p.dq, p.dk, p.dv = dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    _check(_lib.load().eagle_attn_bwd_noalloc(ctypes.byref(p), _stream()),
           "eagle_attn_bwd_noalloc")
    return dq, dk, dv


def merge_out_lse(out, lse, block_out, block_lse, init=False):
    """In place: (out, lse) <- (out, lse) merged with (block_out, block_lse)
    (or copied from it when ``init``).  out fp32 [B,T,H,D], lse fp32 [B,H,T]."""
    if out.dtype != torch.float32 or lse.dtype != torch.float32 or block_lse.dtype != torch.float32:
        raise TypeError("out, lse and block_lse must be float32")
    for t in (out, lse, block_out, block_lse):
        if not t.is_contiguous():
            raise ValueError("merge operands must be contiguous")
    B, T, H, D = out.shape
    if block_out.shape != out.shape or lse.shape != (B, H, T) or block_lse.shape != lse.shape:
        raise ValueError("shape mismatch")
    _check(_lib.load().attn_merge_out_lse(out.data_ptr(), lse.data_ptr(), block_out.data_ptr(),
                                          _dt(block_out), block_lse.data_ptr(), B, T, H, D,
                                          1 if init else 0, _stream()), "attn_merge_out_lse")
    return out, lse


def merge_diag(out, lse, q, cache_k, cache_v, scale=None):
    """In place: fold the diagonal blocks 1..NB-1 into the fp32 running
    (out, lse) of query rows q."""
    p, _ = _params(q, cache_k, cache_v, scale, None, None, 0, 0, True, "generic")
    if out.dtype != torch.float32 or not _same_layout(out, q):
        raise ValueError("out must be float32 with q's strides")
    p.out_dtype = F32
    p.out, p.lse = out.data_ptr(), lse.data_ptr()
    _check(_lib.load().attn_merge_diag(ctypes.byref(p), _stream()), "attn_merge_diag")
    return out, lse


def finalize(src: torch.Tensor, dtype: torch.dtype, out: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 running output -> ``dtype`` (into ``out`` if given, else a new
    contiguous tensor).  With dtype float32 it is a plain copy."""
    if src.dtype != torch.float32 or not src.is_contiguous():
        raise ValueError("src must be a contiguous float32 tensor")
    if out is None:
        out = torch.empty(src.shape, dtype=dtype, device=src.device)
    if out.dtype != dtype or not out.is_contiguous() or out.numel() != src.numel():
        raise ValueError("out must be a contiguous tensor of dtype with src's size")
    dst = out
    _check(_lib.load().attn_finalize(src.data_ptr(), dst.data_ptr(), _dt(dst), src.numel(),
                                     _stream()), "attn_finalize")
    return dst


def launch_count() -> int:
    """Kernels launched by libeagleattn so far in this process."""
    return int(_lib.load().eagle_attn_launch_count())


def selftest_wait_timeout(limit_ns: int = 10_000_000) -> None:
    """Enqueue the bounded-wait self-test (eagle_attn_selftest_wait_timeout):
    after it runs, get_status() reports EAGLE_ATTN_DEV_TIMEOUT (4)."""
    _check(_lib.load().eagle_attn_selftest_wait_timeout(int(limit_ns), _stream()),
           "eagle_attn_selftest_wait_timeout")


def get_status() -> int:
    code = ctypes.c_int(0)
    _check(_lib.load().eagle_attn_get_status(ctypes.byref(code)), "eagle_attn_get_status")
    return code.value


def clear_status() -> None:
    _check(_lib.load().eagle_attn_clear_status(), "eagle_attn_clear_status")


class _EagleAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, cache_k, cache_v, scale, cu_seqlens, max_seqlen):
        out, lse = fwd(q, cache_k, cache_v, scale, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen)
        ctx.save_for_backward(q, cache_k, cache_v, out, lse)
        ctx.scale, ctx.cu, ctx.max_seqlen = scale, cu_seqlens, max_seqlen
        return out

    @staticmethod
    def backward(ctx, grad_out):
        q, k, v, out, lse = ctx.saved_tensors
        if not _same_layout(grad_out, q):
            raise ValueError("grad_out must have q's layout")
        dq, dk, dv = bwd(grad_out, q, k, v, out, lse, ctx.scale, cu_seqlens=ctx.cu,
                         max_seqlen=ctx.max_seqlen)
        return dq, dk, dv, None, None, None


def eagle_attention(q, cache_k, cache_v, scale=None, cu_seqlens=None, max_seqlen=None):
    """Differentiable mixed attention (cf. cached_ring_attention /
    cached_ulysses_attention on a single GPU): q [B,T,H,D], cache_k/cache_v
    stacked [B,NB,T,H,D].  Returns out [B,T,H,D] in q's dtype."""
    return _EagleAttention.apply(q, cache_k, cache_v, scale, cu_seqlens, max_seqlen)
