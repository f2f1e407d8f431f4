"""Sequence-parallel zig-zag ring over torch.distributed ranks.

NeMo AutoModel "eagle.zigzag_ring_attention" (module docstring) and
"eagle.ring_attention" (_CachedZigZagRingAttention): the sequence is cut into
2*cp chunks of c rows; rank r of the cp ranks holds chunk r (early) and chunk
2*cp-1-r (late) of q, of every cache block and of the gradients, concatenated
into a local shard of 2c rows.  Block 0 needs the keys of every earlier chunk,
so the block-0 K/V shards travel around the ring: at step s rank r holds the
shard of rank (r - s) mod cp and attends each of its query chunks to each
visiting key chunk at or before it, with global positions.  The per-pair
results are merged by the log-sum-exp identity in fp32 (_update_out_and_lse);
the diagonal blocks (i >= 1) are per position, so they stay local and are
merged once at the end (_merge_diag), before the cast to q's dtype.

The backward ("eagle.zigzag_ring_attention", zigzag_ring_flash_attn_varlen_
backward) runs every such pair against the FINAL merged out / lse of the
query rows.  dQ accumulates locally; the dK / dV running sums of a block-0
shard travel the ring one step behind its K/V, in fp32, and make the whole
circle (cp hops), so that every rank's sum comes home holding the
contributions of all ranks.  A rank computes its contribution to the visiting
shard into a zeroed buffer while that shard's running sum is still in flight
from the previous rank, and adds it on arrival before passing the sum on: the
hop overlaps the step's compute.  The diagonal blocks' gradients are local and
closed form; they come with the pairs on the diagonal.

Every compute step is one of five operations (``ops``): the default,
``LIBRARY_OPS``, calls libeagleattn (eagle_attn_fwd / eagle_attn_bwd with
global offsets, attn_merge_out_lse, attn_merge_diag, attn_finalize); a caller
may pass another object with the same five methods.  Communication is
torch.distributed point-to-point (batch_isend_irecv: NCCL over NVLink between
GPUs, or any backend that supports it); the K/V exchange is posted before the
step's compute, so that the transfer overlaps it.  Between two ranks the
messages of the two streams (K/V, and the backward's running sums) are posted
in the same order on both sides: every rank posts a step's receive of a
running sum before that step's K/V exchange and sends its updated sum after
the step's compute.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import bwd as _bwd
from . import bwd_workspace_size as _bwd_ws
from . import finalize as _finalize
from . import fwd as _fwd
from . import merge_diag as _merge_diag
from . import merge_out_lse as _merge_out_lse


class LibraryOps:
    """The ring's compute steps as calls into libeagleattn."""

    def __init__(self, impl: str = "auto"):
        self.impl = impl
        self._ws = None

    def fwd_block(self, q, k, v, scale, q_pos_offset, k_pos_offset, out, lse):
        """Block-0 attention of q to k / v (one cache block) with global
        positions, written unrounded: out fp32 [1, c, H, D], lse [1, H, c]."""
        _fwd(q, k, v, scale, q_pos_offset=q_pos_offset, k_pos_offset=k_pos_offset,
             out_dtype=torch.float32, impl=self.impl, out=out, lse=lse)

    def merge(self, out, lse, block_out, block_lse):
        _merge_out_lse(out, lse, block_out, block_lse)

    def merge_diag(self, out, lse, q, cache_k, cache_v, scale):
        _merge_diag(out, lse, q, cache_k, cache_v, scale)

    def finalize(self, src, dtype, out):
        _finalize(src, dtype, out=out)

    def bwd_pair(self, dout, q, k, v, out, lse, scale, q_pos_offset, k_pos_offset, dq, dk, dv):
        """Gradients of one (query chunk, key chunk) pair against the merged
        out / lse, added into the fp32 dq / dk / dv (k / v carry block 0 only,
        or every block when the key chunk is the query chunk)."""
        need = max(1, _bwd_ws(q, k, v, scale=scale, impl=self.impl))
        if self._ws is None or self._ws.numel() < need or self._ws.device != q.device:
            self._ws = torch.empty(need, dtype=torch.uint8, device=q.device)
        _bwd(dout, q, k, v, out, lse, scale, q_pos_offset=q_pos_offset,
             k_pos_offset=k_pos_offset, impl=self.impl, workspace=self._ws, dq=dq, dk=dk, dv=dv,
             grad_accumulate=True)


LIBRARY_OPS = LibraryOps()


def zigzag_shard(x: torch.Tensor, rank: int, cp: int, dim: int) -> torch.Tensor:
    """Rank ``rank``'s zig-zag shard of ``x`` along ``dim``: chunks rank and
    2*cp-1-rank of 2*cp equal chunks, concatenated (a copy)."""
    c = x.shape[dim] // (2 * cp)
    if x.shape[dim] != 2 * cp * c:
        raise ValueError("the sharded length must be divisible by 2*cp")
    a, b = rank, 2 * cp - 1 - rank
    return torch.cat([x.narrow(dim, a * c, c), x.narrow(dim, b * c, c)], dim=dim)


def zigzag_unshard(shards, dim: int) -> torch.Tensor:
    """The whole sequence from the zig-zag shards of all ranks (``shards[r]``
    is rank r's, as zigzag_shard cuts it): the inverse of zigzag_shard."""
    cp = len(shards)
    if cp < 1 or any(x.shape != shards[0].shape for x in shards):
        raise ValueError("one shard per rank, all of the same shape")
    c2 = shards[0].shape[dim]
    if c2 % 2:
        raise ValueError("a zig-zag shard holds two chunks of equal length")
    c = c2 // 2
    chunks = [None] * (2 * cp)
    for r, x in enumerate(shards):
        chunks[r] = x.narrow(dim, 0, c)
        chunks[2 * cp - 1 - r] = x.narrow(dim, c, c)
    return torch.cat(chunks, dim=dim)


def _ring(group):
    cp = dist.get_world_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % cp) if group is not None else (r + 1) % cp
    prv = dist.get_global_rank(group, (r - 1) % cp) if group is not None else (r - 1) % cp
    return r, cp, nxt, prv


def _exchange(send: list[torch.Tensor], recv: list[torch.Tensor], nxt: int, prv: int, group):
    """Posts the sends of ``send`` to the next rank and the receives of ``recv``
    from the previous one; returns the works to wait on."""
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, prv, group) for t in recv]
    return dist.batch_isend_irecv(ops) if ops else []


def _pairs(r: int, src: int, cp: int):
    """(local query chunk slot, query chunk, local key chunk slot, key chunk)
    for the pairs rank r computes against rank src's shard: key chunk at or
    before the query chunk."""
    qch = (r, 2 * cp - 1 - r)
    kch = (src, 2 * cp - 1 - src)
    return [(qi, qc, ki, kc) for qi, qc in enumerate(qch) for ki, kc in enumerate(kch) if kc <= qc]


def ring_zigzag_forward(q, cache_k, cache_v, scale, group=None, ops=None):
    """Forward of the joint softmax on this rank's zig-zag shard.

    q [1, 2c, H, D] and cache_k / cache_v [1, NB, 2c, H, D]: this rank's
    shard (zigzag_shard of the whole sequence along the row dim), the same c
    on every rank.  Collective over ``group`` (default: the world): every rank
    calls it with its own shard.  Returns (out [1, 2c, H, D] in q's dtype,
    lse [1, H, 2c] fp32) of the local rows, equal to those rows of the
    unsharded forward."""
    ops = LIBRARY_OPS if ops is None else ops
    B, T2, H, D = q.shape
    if B != 1 or T2 % 2 or cache_k.shape[2] != T2 or cache_v.shape != cache_k.shape:
        raise ValueError("a zig-zag shard is [1, 2c, H, D] with a [1, NB, 2c, H, D] cache")
    c = T2 // 2
    r, cp, nxt, prv = _ring(group)
    f32 = dict(dtype=torch.float32, device=q.device)
    o_run = [torch.zeros((1, c, H, D), **f32) for _ in range(2)]
    l_run = [torch.full((1, H, c), -float("inf"), **f32) for _ in range(2)]
    blk_o = torch.empty((1, c, H, D), **f32)
    blk_l = torch.empty((1, H, c), **f32)
    kv = [cache_k[:, :1].contiguous(), cache_v[:, :1].contiguous()]
    kv_next = [torch.empty_like(kv[0]), torch.empty_like(kv[1])] if cp > 1 else None
    for s in range(cp):
        src = (r - s) % cp
        works = _exchange(kv, kv_next, nxt, prv, group) if s + 1 < cp else []
        for qi, qc, ki, kc in _pairs(r, src, cp):
            ops.fwd_block(q[:, qi * c:(qi + 1) * c], kv[0][:, :, ki * c:(ki + 1) * c],
                          kv[1][:, :, ki * c:(ki + 1) * c], scale, qc * c, kc * c, blk_o, blk_l)
            ops.merge(o_run[qi], l_run[qi], blk_o, blk_l)
        for w in works:
            w.wait()
        if works:
            kv, kv_next = kv_next, kv
    out = torch.empty_like(q)
    lse = torch.empty((1, H, T2), **f32)
    for qi in range(2):
        rows = slice(qi * c, (qi + 1) * c)
        ops.merge_diag(o_run[qi], l_run[qi], q[:, rows], cache_k[:, :, rows], cache_v[:, :, rows],
                       scale)
        ops.finalize(o_run[qi], q.dtype, out[:, rows])
        for h in range(H):  # one contiguous run of lse per head
            ops.finalize(l_run[qi][0, h], torch.float32, lse[0, h, rows])
    return out, lse


def ring_zigzag_backward(grad_out, q, cache_k, cache_v, out, lse, scale, group=None, ops=None):
    """Backward of the joint softmax on this rank's zig-zag shard.

    Shards as ring_zigzag_forward; out / lse are this rank's rows of the
    merged forward (ring_zigzag_forward's results).  Collective over
    ``group``.  Returns (dq [1, 2c, H, D], dk / dv [1, NB, 2c, H, D]) in q's
    dtype: this rank's rows of the unsharded gradients."""
    ops = LIBRARY_OPS if ops is None else ops
    B, T2, H, D = q.shape
    if B != 1 or T2 % 2 or cache_k.shape[2] != T2 or cache_v.shape != cache_k.shape:
        raise ValueError("a zig-zag shard is [1, 2c, H, D] with a [1, NB, 2c, H, D] cache")
    c = T2 // 2
    r, cp, nxt, prv = _ring(group)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq32 = torch.zeros(q.shape, **f32)
    dk32 = torch.zeros(cache_k.shape, **f32)  # this shard's blocks (block 0: its own part first)
    dv32 = torch.zeros(cache_k.shape, **f32)
    lse_c = [lse[:, :, qi * c:(qi + 1) * c].contiguous() for qi in range(2)]
    kv = [cache_k[:, :1].contiguous(), cache_v[:, :1].contiguous()]
    kv_next = [torch.empty_like(kv[0]), torch.empty_like(kv[1])] if cp > 1 else None
    acc_shape = (1, 1, T2, H, D)
    # this rank's part of the visiting shard's block-0 dK / dV (steps s >= 1), and
    # two buffers for the running sums that arrive, one per step parity: a sum is
    # received, completed and sent on from the same buffer
    part = [torch.empty(acc_shape, **f32) for _ in range(2)] if cp > 1 else None
    inbox = [[torch.empty(acc_shape, **f32) for _ in range(2)] for _ in range(2)] \
        if cp > 1 else None
    sending = [[], []]  # the works of the send out of inbox[0] / inbox[1] (or of step 0)
    for s in range(cp):
        src = (r - s) % cp
        # the running sum of shard src (the previous rank's step s-1), then this step's K/V
        box = inbox[s & 1] if s > 0 else None
        if s > 0:
            for w in sending[s & 1]:  # the buffer's last send has left it
                w.wait()
            sending[s & 1] = []
        recv_works = _exchange([], box, nxt, prv, group) if s > 0 else []
        works = _exchange(kv, kv_next, nxt, prv, group) if s + 1 < cp else []
        if s == 0:
            acc = [dk32[:, :1], dv32[:, :1]]
        else:
            for t in part:
                t.zero_()
            acc = part
        for qi, qc, ki, kc in _pairs(r, src, cp):
            qrows = slice(qi * c, (qi + 1) * c)
            krows = slice(ki * c, (ki + 1) * c)
            if s == 0 and kc == qc:
                # the pair on the diagonal carries the diagonal blocks (local)
                kk, vv = cache_k[:, :, qrows], cache_v[:, :, qrows]
                dkk, dvv = dk32[:, :, qrows], dv32[:, :, qrows]
            else:
                kk, vv = kv[0][:, :, krows], kv[1][:, :, krows]
                dkk, dvv = acc[0][:, :, krows], acc[1][:, :, krows]
            ops.bwd_pair(grad_out[:, qrows], q[:, qrows], kk, vv, out[:, qrows], lse_c[qi], scale,
                         qc * c, kc * c, dq32[:, qrows], dkk, dvv)
        for w in works:
            w.wait()
        if cp > 1:
            if s == 0:
                out_sum = acc  # this shard's own part starts its circle
            else:
                for w in recv_works:
                    w.wait()
                box[0].add_(part[0])
                box[1].add_(part[1])
                out_sum = box
            sending[s & 1] = _exchange(out_sum, [], nxt, prv, group)
            if s + 1 < cp:
                kv, kv_next = kv_next, kv
    if cp > 1:
        # after cp hops the running sums of this rank's own shard are home
        home = [torch.empty(acc_shape, **f32) for _ in range(2)]
        for w in _exchange([], home, nxt, prv, group):
            w.wait()
        for ws in sending:
            for w in ws:
                w.wait()
        dk32[:, :1].copy_(home[0])
        dv32[:, :1].copy_(home[1])
    dq = torch.empty_like(q)
    dk = torch.empty_like(cache_k)
    dv = torch.empty_like(cache_v)
    ops.finalize(dq32, q.dtype, dq)
    for i in range(cache_k.shape[1]):
        ops.finalize(dk32[:, i], q.dtype, dk[:, i])
        ops.finalize(dv32[:, i], q.dtype, dv[:, i])
    return dq, dk, dv
