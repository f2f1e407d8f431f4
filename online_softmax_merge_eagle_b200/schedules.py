"""Chunk schedules of the context-parallel variants, emulated on one GPU.

NeMo AutoModel "eagle.zigzag_ring_attention" (module docstring): the sequence
is cut into 2*cp chunks and rank r owns chunk r (early) and chunk 2*cp-1-r
(late); each rank attends its query chunks to every key chunk that precedes
them (causally, with global positions) and merges the per-chunk results with
the online-softmax log-sum-exp identity; the per-position diagonals (blocks
i >= 1) are layout agnostic and merge unchanged ("eagle.ring_attention",
_CachedZigZagRingAttention).

With packed documents ("eagle.zigzag_ring_attention", module text: varlen
throughout; get_half_index / get_half_lse select the front and back half of
every document) every DOCUMENT is cut into 2*cp chunks and rank r owns chunk
r and chunk 2*cp-1-r of each of them; documents never attend to each other,
so the varlen schedule is the per-document schedule, document by document.

The backward of the same schedule ("eagle.zigzag_ring_attention",
zigzag_ring_flash_attn_varlen_backward; "eagle.ulysses_attention",
_block0_backward) runs every (query chunk, key chunk <= query chunk) pair
against the FINAL merged out / lse of the query chunk: the pair's dq adds into
the query chunk's gradient and its dk / dv into the key chunk's block-0
gradient; the pair on the diagonal also carries the diagonal blocks, whose
grads are closed form per row.

Here every step of that schedule is a call into the library: the per-chunk
block-0 forward (eagle_attn_fwd with global offsets, fp32 block output),
attn_merge_out_lse, attn_merge_diag, the per-pair backward (eagle_attn_bwd
with global offsets, gradients added into fp32 buffers) and attn_finalize.
This module only orders the calls and slices views; it computes nothing
itself.
"""
from __future__ import annotations

import torch

from . import bwd, bwd_workspace_size, finalize, fwd, merge_diag, merge_out_lse, query_segments


def zigzag_owner_chunks(rank: int, cp: int) -> tuple[int, int]:
    """(early, late) chunk indices held by ``rank`` (rank r: r and 2cp-1-r)."""
    return rank, 2 * cp - 1 - rank


def zigzag_forward(q, cache_k, cache_v, scale, cp: int, impl: str = "auto", out=None, lse=None,
                   ranks=None, single_launch: bool = False):
    """Forward of the whole sequence through the zig-zag chunk schedule.

    q [1, T, H, D], cache_k / cache_v [1, NB, T, H, D] (B = 1, as the zig-zag
    ring is varlen and unbatched); T must be a multiple of 2*cp.  Every emulated
    rank (or the ranks listed in ``ranks``) processes its two query chunks:
    block-0 attention to each key chunk at or before the query chunk, merged in
    fp32, then the diagonal blocks, then the cast to q's dtype.  Returns
    (out [1, T, H, D] q dtype, lse [1, H, T] fp32); rows of ranks not listed are
    left untouched.  ``single_launch``: one forward launch per rank over its
    query tiles against every key, the key chunks merged inside the kernel (chunk
    length a multiple of 128).
    """
    return _chunk_schedule_forward(q, cache_k, cache_v, scale, 2 * cp,
                                   [zigzag_owner_chunks(r, cp)
                                    for r in (range(cp) if ranks is None else ranks)],
                                   impl, out, lse, single_launch)


def contiguous_forward(q, cache_k, cache_v, scale, cp: int, impl: str = "auto", out=None,
                       lse=None, ranks=None, single_launch: bool = False):
    """Forward through the contiguous ring ("eagle.ring_attention", module text:
    rank r owns chunk r of cp; at ring step s <= r it sees the key chunk r - s,
    causally only at step 0).  Arguments as zigzag_forward; T a multiple of cp."""
    return _chunk_schedule_forward(q, cache_k, cache_v, scale, cp,
                                   [(r,) for r in (range(cp) if ranks is None else ranks)],
                                   impl, out, lse, single_launch)


def _chunk_schedule_forward(q, cache_k, cache_v, scale, n_chunks, rank_chunks, impl, out, lse,
                            single_launch):
    B, T, H, D = q.shape
    if B != 1 or T % n_chunks:
        raise ValueError("chunk schedules need B == 1 and T divisible by the chunk count")
    c = T // n_chunks
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((1, H, T), dtype=torch.float32, device=q.device)
    if single_launch:
        if c % 128:
            raise ValueError("single_launch needs chunks of a multiple of 128 rows")
        for chunks in rank_chunks:
            # the rank's 128-row tiles, latest (heaviest) first
            rows = [t for ch in sorted(chunks, reverse=True)
                    for t in range(ch * c + c - 128, ch * c - 1, -128)]
            tiles = torch.tensor(rows, dtype=torch.int32).to(q.device, non_blocking=True)
            fwd(q, cache_k, cache_v, scale, impl=impl, out=out, lse=lse, q_tiles=tiles)
        return out, lse
    o_run = torch.empty((1, c, H, D), dtype=torch.float32, device=q.device)
    l_run = torch.empty((1, H, c), dtype=torch.float32, device=q.device)
    blk_o = torch.empty((1, c, H, D), dtype=torch.float32, device=q.device)
    blk_l = torch.empty((1, H, c), dtype=torch.float32, device=q.device)
    k0, v0 = cache_k[:, :1], cache_v[:, :1]
    for chunks in rank_chunks:
        for qc in chunks:
            qs = slice(qc * c, (qc + 1) * c)
            for kc in range(qc + 1):  # key chunks after the query chunk are fully masked
                ks = slice(kc * c, (kc + 1) * c)
                dst_o, dst_l = (o_run, l_run) if kc == 0 else (blk_o, blk_l)
                fwd(q[:, qs], k0[:, :, ks], v0[:, :, ks], scale, q_pos_offset=qc * c,
                    k_pos_offset=kc * c, out_dtype=torch.float32, impl=impl, out=dst_o, lse=dst_l)
                if kc > 0:
                    merge_out_lse(o_run, l_run, blk_o, blk_l)
            merge_diag(o_run, l_run, q[:, qs], cache_k[:, :, qs], cache_v[:, :, qs], scale)
            finalize(o_run, q.dtype, out=out[:, qs])
            for h in range(H):  # lse rows of this chunk, one contiguous run per head
                finalize(l_run[0, h], torch.float32, out=lse[0, h, qs])
    return out, lse


def zigzag_rank_rows(rank: int, cp: int, a: int, b: int) -> list[tuple[int, int]]:
    """Half-open row ranges of ``rank``'s two chunks of the sequence [a, b) cut into
    2*cp chunks ("eagle.zigzag_ring_attention", get_half_index: the front and
    back half that rank r holds)."""
    c = (b - a) // (2 * cp)
    return [(a + ch * c, a + (ch + 1) * c) for ch in zigzag_owner_chunks(rank, cp)]


def _single_launch_backward(grad_out, q, cache_k, cache_v, out, lse, scale, rank_rows, impl,
                            dq32, dk32, dv32, **mask):
    """One backward launch per emulated rank over its query rows (every key
    they see, in one kernel), summed into fp32 buffers."""
    for rows in rank_rows:
        tiles, counts = query_segments(rows, q.device)
        bwd(grad_out, q, cache_k, cache_v, out, lse, scale, impl=impl, dq=dq32, dk=dk32, dv=dv32,
            grad_accumulate=True, q_tiles=tiles, q_tile_rows=counts, **mask)


def zigzag_backward(grad_out, q, cache_k, cache_v, out, lse, scale, cp: int, impl: str = "auto",
                    dq=None, dk=None, dv=None, ranks=None, acc32=None, deterministic=False,
                    single_launch: bool = False):
    """Backward of the whole sequence through the zig-zag chunk schedule.

    Shapes as zigzag_forward; out / lse are the merged forward results of the
    whole sequence (from zigzag_forward or an unchunked forward).  Every
    emulated rank (or those in ``ranks``) runs, for each of its query chunks,
    one backward per key chunk at or before it: block 0 only below the
    diagonal, block 0 plus the diagonal blocks on it.  Gradients accumulate in
    fp32 and are cast to q's dtype at the end.  Returns (dq, dk, dv); only the
    contributions of the listed ranks are included.  ``acc32`` = (dq32, dk32,
    dv32): zeroed fp32 accumulators with q's / cache_k's element strides to use
    instead of fresh ones (the varlen schedule passes views of whole-sequence
    buffers).  ``deterministic`` selects the reproducible backward for every
    pair (eagle_attn_params.deterministic).  ``single_launch``: one backward
    launch per rank over its two query chunks against every key (a segment list
    in the ABI), instead of one call per chunk pair; not with ``deterministic``.
    """
    B, T, H, D = q.shape
    if B != 1 or T % (2 * cp):
        raise ValueError("zig-zag schedule needs B == 1 and T divisible by 2*cp")
    c = T // (2 * cp)
    f32 = dict(dtype=torch.float32, device=q.device)
    if acc32 is None:
        acc32 = (torch.zeros(q.shape, **f32), torch.zeros(cache_k.shape, **f32),
                 torch.zeros(cache_k.shape, **f32))
    dq32, dk32, dv32 = acc32
    if single_launch:
        if deterministic:
            raise ValueError("the single-launch backward is the five-product kernel only")
        _single_launch_backward(grad_out, q, cache_k, cache_v, out, lse, scale,
                                [zigzag_rank_rows(r, cp, 0, T)
                                 for r in (range(cp) if ranks is None else ranks)],
                                impl, dq32, dk32, dv32)
        return _finalize_grads(q, cache_k, dq32, dk32, dv32, dq, dk, dv)
    lse_c = torch.empty((1, H, c), **f32)
    k0, v0 = cache_k[:, :1], cache_v[:, :1]
    ws = torch.empty(max(1, bwd_workspace_size(q[:, :c], cache_k[:, :, :c], cache_v[:, :, :c],
                                               scale=scale, impl=impl)),
                     dtype=torch.uint8, device=q.device)
    for r in (range(cp) if ranks is None else ranks):
        for qc in zigzag_owner_chunks(r, cp):
            qs = slice(qc * c, (qc + 1) * c)
            for h in range(H):  # the query chunk's merged lse rows, contiguous per head
                finalize(lse[0, h, qs], torch.float32, out=lse_c[0, h])
            for kc in range(qc + 1):  # key chunks after the query chunk are fully masked
                if kc < qc:
                    ks = slice(kc * c, (kc + 1) * c)
                    kk, vv, dkk, dvv = k0[:, :, ks], v0[:, :, ks], dk32[:, :1, ks], dv32[:, :1, ks]
                else:
                    kk, vv = cache_k[:, :, qs], cache_v[:, :, qs]
                    dkk, dvv = dk32[:, :, qs], dv32[:, :, qs]
                bwd(grad_out[:, qs], q[:, qs], kk, vv, out[:, qs], lse_c, scale,
                    q_pos_offset=qc * c, k_pos_offset=kc * c, impl=impl, workspace=ws,
                    dq=dq32[:, qs], dk=dkk, dv=dvv, grad_accumulate=True,
                    deterministic=deterministic)
    return _finalize_grads(q, cache_k, dq32, dk32, dv32, dq, dk, dv)


def _finalize_grads(q, cache_k, dq32, dk32, dv32, dq, dk, dv):
    """The fp32 sums cast to q's dtype (into dq / dk / dv when given)."""
    dq = finalize(dq32, q.dtype, out=dq)
    if dk is None:
        dk = torch.empty_like(cache_k)
    if dv is None:
        dv = torch.empty_like(cache_k)
    for i in range(cache_k.shape[1]):  # block by block: dk / dv may be views of a larger cache
        finalize(dk32[:, i], q.dtype, out=dk[:, i])
        finalize(dv32[:, i], q.dtype, out=dv[:, i])
    return dq, dk, dv


def _doc_bounds(cu_seqlens, T: int, cp: int) -> list[tuple[int, int]]:
    cu = [int(x) for x in (cu_seqlens.tolist() if isinstance(cu_seqlens, torch.Tensor)
                           else list(cu_seqlens))]
    if cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must run from 0 to T, non-decreasing")
    docs = [(a, b) for a, b in zip(cu, cu[1:]) if b > a]
    if any((b - a) % (2 * cp) for a, b in docs):
        raise ValueError("every document length must be divisible by 2*cp (zig-zag halves)")
    return docs


def _packed_mask(cu_seqlens, T, device):
    """cu_seqlens as a device int32 tensor and the longest document."""
    cu = [int(x) for x in (cu_seqlens.tolist() if isinstance(cu_seqlens, torch.Tensor)
                           else list(cu_seqlens))]
    return (torch.tensor(cu, dtype=torch.int32).to(device, non_blocking=True),
            max(b - a for a, b in zip(cu, cu[1:])))


def varlen_zigzag_forward(q, cache_k, cache_v, scale, cu_seqlens, cp: int, impl: str = "auto",
                          out=None, lse=None, single_launch: bool = False, ranks=None):
    """Forward of packed documents through the varlen zig-zag schedule: each
    document's 2*cp chunks through zigzag_forward (the document's positions
    start at 0, so no mask crosses documents).  q [1, T, H, D], cache_k/cache_v
    [1, NB, T, H, D]; cu_seqlens (host sequence or tensor) [num_docs + 1] with
    every length divisible by 2*cp.  Returns (out, lse) like zigzag_forward.
    ``single_launch``: one launch per emulated rank (or the ``ranks`` listed)
    over its front and back chunk of every document at once, the packed
    (cu_seqlens) mask keeping the documents apart -- the pages' one varlen call
    per ring step over every document's halves."""
    B, T, H, D = q.shape
    if B != 1:
        raise ValueError("the varlen zig-zag schedule is unbatched (B == 1)")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((1, H, T), dtype=torch.float32, device=q.device)
    docs = _doc_bounds(cu_seqlens, T, cp)
    if single_launch:
        cu_d, max_len = _packed_mask(cu_seqlens, T, q.device)
        for r in (range(cp) if ranks is None else ranks):
            tiles, counts = query_segments([rr for a, b in docs
                                            for rr in zigzag_rank_rows(r, cp, a, b)], q.device)
            fwd(q, cache_k, cache_v, scale, cu_seqlens=cu_d, max_seqlen=max_len, impl=impl,
                out=out, lse=lse, q_tiles=tiles, q_tile_rows=counts)
        return out, lse
    for a, b in docs:
        zigzag_forward(q[:, a:b], cache_k[:, :, a:b], cache_v[:, :, a:b], scale, cp, impl=impl,
                       out=out[:, a:b], lse=lse[:, :, a:b])
    return out, lse


def varlen_zigzag_backward(grad_out, q, cache_k, cache_v, out, lse, scale, cu_seqlens, cp: int,
                           impl: str = "auto", dq=None, dk=None, dv=None, deterministic=False,
                           single_launch: bool = False):
    """Backward of the varlen zig-zag schedule: each document's chunk pairs
    through zigzag_backward against the document's merged out / lse rows.
    Returns (dq, dk, dv) in q's dtype.  ``single_launch``: one backward launch
    per emulated rank over its chunks of every document (packed mask), the
    ranks' parts summed in fp32; not with ``deterministic``."""
    B, T, H, D = q.shape
    if B != 1:
        raise ValueError("the varlen zig-zag schedule is unbatched (B == 1)")
    if dq is None:
        dq = torch.empty_like(q)
    if dk is None:
        dk = torch.empty_like(cache_k)
    if dv is None:
        dv = torch.empty_like(cache_v)
    # whole-sequence fp32 accumulators; each document works on its rows of them
    f32 = dict(dtype=torch.float32, device=q.device)
    dq32 = torch.zeros(q.shape, **f32)
    dk32 = torch.zeros(cache_k.shape, **f32)
    dv32 = torch.zeros(cache_k.shape, **f32)
    docs = _doc_bounds(cu_seqlens, T, cp)
    if single_launch:
        if deterministic:
            raise ValueError("the single-launch backward is the five-product kernel only")
        cu_d, max_len = _packed_mask(cu_seqlens, T, q.device)
        _single_launch_backward(grad_out, q, cache_k, cache_v, out, lse, scale,
                                [[rr for a, b in docs for rr in zigzag_rank_rows(r, cp, a, b)]
                                 for r in range(cp)],
                                impl, dq32, dk32, dv32, cu_seqlens=cu_d, max_seqlen=max_len)
        return _finalize_grads(q, cache_k, dq32, dk32, dv32, dq, dk, dv)
    for a, b in docs:
        zigzag_backward(grad_out[:, a:b], q[:, a:b], cache_k[:, :, a:b], cache_v[:, :, a:b],
                        out[:, a:b], lse[:, :, a:b], scale, cp, impl=impl, dq=dq[:, a:b],
                        dk=dk[:, :, a:b], dv=dv[:, :, a:b],
                        acc32=(dq32[:, a:b], dk32[:, :, a:b], dv32[:, :, a:b]),
                        deterministic=deterministic)
    return dq, dk, dv
