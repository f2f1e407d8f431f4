"""The library's mask range functions against brute-force visibility (CPU).

The kernels never test a (row, key) pair outside the row and key ranges these
functions return, and the backward derives each key's visible rows from
``key_rows``, so a range that is too short drops gradient terms.  The visibility
rule restated here is the one the kernels implement: block-0 key s is visible to
query row t iff both global positions lie in the same packed document
(``cu_seqlens``) and, when causal, k_pos <= q_pos (NeMo AutoModel
"eagle.ulysses_attention", _block0_forward and attach_cp_kv_gather_hooks).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    if not os.path.exists(NVCC) and shutil.which("nvcc") is None:
        pytest.fail("nvcc is needed to build the host harness of the mask functions")
    exe = str(tmp_path_factory.mktemp("mask") / "mask_ranges")
    subprocess.check_call([NVCC if os.path.exists(NVCC) else "nvcc", "-std=c++17", "-O1",
                           "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", os.path.join(os.path.dirname(HERE), "include"),
                           "-o", exe, os.path.join(HERE, "mask_ranges_host.cu")])
    return exe


def visibility(Tq, Tk, q_off, k_off, causal, cu):
    qp = q_off + np.arange(Tq)[:, None]
    kp = k_off + np.arange(Tk)[None, :]
    vis = np.ones((Tq, Tk), dtype=bool)
    if causal:
        vis &= kp <= qp
    if cu is not None:
        cu = np.asarray(cu, dtype=np.int64)

        def doc(pos):
            d = np.searchsorted(cu, pos, side="right") - 1
            return np.where((pos < 0) | (pos >= cu[-1]), -1, d)

        dq, dk = doc(qp), doc(kp)
        vis &= (dq == dk) & (dq >= 0)
    return vis


def span(mask_1d):
    """(first, last) index of a 1-D boolean mask, checking it is one run; None if empty."""
    idx = np.flatnonzero(mask_1d)
    if idx.size == 0:
        return None
    assert idx[-1] - idx[0] + 1 == idx.size, "visible set is not one interval"
    return int(idx[0]), int(idx[-1])


def run(harness, Tq, Tk, q_off, k_off, causal, cu):
    nd = 0 if cu is None else len(cu) - 1
    text = f"{Tq} {Tk} {q_off} {k_off} {int(causal)} {nd}"
    if cu is not None:
        text += " " + " ".join(str(int(x)) for x in cu)
    out = subprocess.run([harness], input=text, capture_output=True, text=True, check=True).stdout
    return [line.split() for line in out.splitlines()]


def doc_cu(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


rng = np.random.default_rng(7)
_lens = rng.integers(1, 90, size=40)
_lens[[3, 11, 12]] = [1, 0, 2]  # a one-token and an empty document
CASES = {
    "causal": (700, 700, 0, 0, True, None),
    "causal_q_after_keys": (300, 900, 500, 0, True, None),
    "causal_q_before_keys": (300, 400, 0, 350, True, None),
    "full": (257, 300, 0, 0, False, None),
    "docs_causal": (int(_lens.sum()), int(_lens.sum()), 0, 0, True, doc_cu(_lens)),
    "docs_query_shard": (400, int(_lens.sum()), 900, 0, True, doc_cu(_lens)),
    "docs_offsets_past_end": (500, 700, -50, 120, True, doc_cu(_lens)),
    "docs_full": (600, 650, 30, 10, False, doc_cu(_lens)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_mask_ranges_match_brute_force(harness, case):
    Tq, Tk, q_off, k_off, causal, cu = CASES[case]
    vis = visibility(Tq, Tk, q_off, k_off, causal, cu)
    lines = run(harness, Tq, Tk, q_off, k_off, causal, cu)
    n = {"R": 0, "Q": 0, "K": 0, "S": 0, "G": 0}
    last_cls = -1
    for rec in lines:
        kind, vals = rec[0], [int(x) for x in rec[1:]]
        n[kind] += 1
        if kind == "R":
            t, cls, lo, hi = vals
            sp = span(vis[t])
            if sp is None:
                assert cls != 0 and hi < lo, rec
            else:
                assert (cls, lo, hi) == (0, sp[0], sp[1]), rec
            assert cls >= last_cls, "row classes must be non-decreasing"
            last_cls = cls
        elif kind == "Q":
            t0, t1, a, b = vals
            sp = span(vis[t0:t1 + 1].any(axis=0))
            assert (b < a) if sp is None else ((a, b) == sp), rec
        elif kind == "K":
            k0, k1, a, b = vals
            sp = span(vis[:, k0:k1 + 1].any(axis=1))
            assert (b < a) if sp is None else ((a, b) == sp), rec
        elif kind == "S":
            s, a, b = vals
            sp = span(vis[:, s]) if 0 <= s < Tk else None
            assert (b < a) if sp is None else ((a, b) == sp), rec
    assert n["R"] == Tq and n["S"] == Tk + 2 and n["Q"] > 0 and n["K"] > 0


def test_block_order_is_a_grouped_heaviest_first_bijection(harness):
    """heavy_first maps the blocks of a (tiles x pairs) grid one to one onto
    (tile, pair); within each group of 8 consecutive pairs the tile index never
    decreases with the block's linear index, so a group's heaviest tiles start
    first."""
    lines = [r for r in run(harness, *CASES["causal"]) if r[0] == "G"]
    grids = {}
    for rec in lines:
        nt, npairs, lin, tile, pair = (int(x) for x in rec[1:])
        grids.setdefault((nt, npairs), []).append((lin, tile, pair))
    assert len(grids) == 6
    for (nt, npairs), recs in grids.items():
        assert sorted(r[0] for r in recs) == list(range(nt * npairs))
        assert sorted((t, p) for _, t, p in recs) == [(t, p) for t in range(nt) for p in range(npairs)]
        last = {}
        for lin, tile, pair in sorted(recs):
            group = pair // 8
            assert tile >= last.get(group, 0), (nt, npairs, lin)
            last[group] = tile
