"""The benchmark's work accounting (CPU): the visible-pair count behind every
TFLOP/s figure against closed forms and a brute-force count, and the per-unit
FLOP and byte figures of the roofline entries.

Visibility is the kernels' rule: key s of block 0 is visible to query row t iff
both global positions lie in the same packed document and k_pos <= q_pos
(NeMo AutoModel "eagle.ulysses_attention", _block0_forward and
"eagle.target_cp", attach_cp_kv_gather_hooks).  The FLOP convention counts 4*D
per visible pair forward (Q K^T and P V) and 10*D backward (five products), plus
4*D / 8*D per row and diagonal block.
"""
import importlib.util
import os
from dataclasses import replace

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def workloads():
    from online_softmax_merge_eagle_b200.inputs import WORKLOADS
    return WORKLOADS


def brute_pairs(Tq, Tk, q_off, k_off, lengths):
    qp = q_off + np.arange(Tq)[:, None]
    kp = k_off + np.arange(Tk)[None, :]
    vis = kp <= qp
    if lengths is not None:
        cu = np.concatenate([[0], np.cumsum(lengths)])
        doc = lambda p: np.where((p < 0) | (p >= cu[-1]), -1, np.searchsorted(cu, p, side="right") - 1)  # noqa: E731
        vis &= (doc(qp) == doc(kp)) & (doc(qp) >= 0)
    return int(vis.sum())


def test_dense_pairs_are_the_causal_triangle(bench, workloads):
    w = workloads["dense_bf16"]
    T = w.Tq
    assert bench.visible_pairs(w) == w.B * w.H * T * (T + 1) // 2 == 2_147_745_792


def test_varlen_pairs_are_the_sum_of_document_triangles(bench, workloads):
    w = workloads["varlen_bf16"]
    L = np.asarray(w.doc_lengths, dtype=np.int64)
    assert L.sum() == w.Tq
    assert bench.visible_pairs(w) == w.B * w.H * int((L * (L + 1) // 2).sum())


def test_frozen_target_pairs_see_every_earlier_key(bench, workloads):
    # queries at global positions q_off .. q_off + T - 1 against the keys 0 .. Tk-1
    w = workloads["frozen_target_bf16"]
    per_row = np.minimum(w.q_pos_offset + np.arange(w.Tq), w.tk - 1) + 1
    assert bench.visible_pairs(w) == w.B * w.H * int(per_row.sum())


@pytest.mark.parametrize("q_off,k_off,lengths", [
    (0, 0, None), (37, 0, None), (0, 20, None), (5, 3, (7, 1, 30, 12, 2)),
    (-4, 6, (13, 29, 10)),
])
def test_pairs_match_a_brute_force_count(bench, workloads, q_off, k_off, lengths):
    # rows before the first or past the last document see nothing
    w = replace(workloads["dense_bf16"], B=2, H=3, Tq=50, Tk=None, q_pos_offset=q_off,
                k_pos_offset=k_off, doc_lengths=lengths)
    assert bench.visible_pairs(w) == 2 * 3 * brute_pairs(50, 50, q_off, k_off, lengths)


def test_flops_follow_the_per_pair_and_per_row_convention(bench, workloads):
    w = workloads["dense_bf16"]
    f = bench.flops(w)
    rows = w.B * w.Tq * w.H
    assert f["fwd"] == 4 * w.D * f["pairs"] + 4 * w.D * (w.num_blocks - 1) * rows
    assert f["bwd"] == 10 * w.D * f["pairs"] + 8 * w.D * (w.num_blocks - 1) * rows
    assert f["total"] == f["fwd"] + f["bwd"]
    assert round(f["fwd"] / 1e12, 4) == 1.1015 and round(10 * w.D * f["pairs"] / 1e12, 4) == 2.7491


def test_row_pass_bytes_per_row(bench, workloads):
    # dO, O, q (2D bytes each) + 7 x (k, v read, dk, dv written) + the fp32 dQ
    # accumulator row + lse and D_t: 768 + 7 * 1024 + 512 + 8 = 8,456 bytes on dense_bf16
    w = workloads["dense_bf16"]
    fl = bench.flops(w)
    pk = {"bf16_tflops": 1000.0, "hbm_gbs": 1000.0, "source": "test"}
    kern = {"fwd_ms": 1.0, "bwd_block0_ms": 2.0, "bwd_all_ms": 3.0}
    e = bench.kernel_rooflines(w, fl, kern, pk)
    rows = w.B * w.Tq * w.H
    assert e["bwd_rows"]["achieved"] == pytest.approx(rows * 8456 / 1e-3 / 1e9)
    assert e["bwd_block0"]["achieved"] == pytest.approx(10 * w.D * fl["pairs"] / 2e-3 / 1e12)
    assert e["fwd"]["achieved"] == pytest.approx(fl["fwd"] / 1e-3 / 1e12)
    for k in ("fwd", "bwd_block0", "bwd_rows"):
        assert e[k]["frac"] == pytest.approx(e[k]["achieved"] / e[k]["peak"])
