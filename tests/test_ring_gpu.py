"""The sequence-parallel zig-zag ring (NeMo AutoModel "eagle.zigzag_ring_attention")
through libeagleattn on one GPU.  With one GPU the ring has one rank: its shard is the whole sequence as two chunks and no shard
moves, but every compute step (block forward with global offsets, merges, the
diagonal merge, the per-pair backward into fp32 accumulators, the casts) is the
library's, checked against the fp64 oracle.  The exchange between ranks is
covered by the gloo tests on the CPU."""
import datetime
import os
import tempfile

import pytest
import torch
import torch.distributed as dist

import oracle
from online_softmax_merge_eagle_b200.inputs import make_tensors
from online_softmax_merge_eagle_b200.ring import (ring_zigzag_backward, ring_zigzag_forward,
                                                  zigzag_shard)
from tests._util import TOL, max_abs, to_np

pytestmark = pytest.mark.gpu

TB = TOL[torch.bfloat16]


@pytest.fixture()
def one_rank_group():
    fd, path = tempfile.mkstemp(prefix="ring_store_")
    os.close(fd)
    os.unlink(path)
    dist.init_process_group("gloo", init_method=f"file://{path}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        yield
    finally:
        dist.destroy_process_group()
        if os.path.exists(path):
            os.unlink(path)


@pytest.mark.parametrize("T,NB", [(512, 3), (768, 1)])
def test_one_rank_ring_matches_oracle(one_rank_group, T, NB):
    t = make_tensors(1, T, 2, 128, NB, torch.bfloat16, seed=5, device="cuda")
    q, k, v, do = t["q"], t["cache_k"], t["cache_v"], t["grad_out"]
    scale = 128 ** -0.5
    sh = lambda x, dim: zigzag_shard(x, 0, 1, dim)  # noqa: E731  (one rank: the whole sequence)
    out, lse = ring_zigzag_forward(sh(q, 1), sh(k, 2), sh(v, 2), scale)
    dq, dk, dv = ring_zigzag_backward(sh(do, 1), sh(q, 1), sh(k, 2), sh(v, 2), out, lse, scale)
    torch.cuda.synchronize()
    ro, rl = oracle.fwd(to_np(q), to_np(k), to_np(v), scale)
    rq, rk, rv = oracle.bwd(to_np(q), to_np(k), to_np(v), to_np(do), scale)
    assert max_abs(out, ro) <= TB["out"]
    assert max_abs(lse, rl) <= TB["lse"]
    assert max_abs(dq, rq) <= TB["grad"]
    assert max_abs(dk, rk) <= TB["grad"]
    assert max_abs(dv, rv) <= TB["grad"]
