"""C-ABI checks that need no GPU: the library loads, exports every function
include/eagleattn.h declares, and rejects bad arguments on the host before
any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import online_softmax_merge_eagle_b200 as ea
from online_softmax_merge_eagle_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eagleattn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "defined")))


def test_header_declares_the_binding_exports():
    assert sorted(_lib.EXPORTS) == declared_functions()


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name


def test_abi_version_and_struct_size():
    lib = _lib.load()
    assert lib.eagle_attn_abi_version() == _lib.ABI_VERSION
    p = _lib.Params()
    lib.eagle_attn_params_init(ctypes.byref(p))
    assert p.struct_size == ctypes.sizeof(_lib.Params)
    assert p.abi_version == _lib.ABI_VERSION
    assert p.causal == 1 and p.impl == 0 and p.dtype == _lib.BF16


def _valid_params():
    lib = _lib.load()
    p = _lib.Params()
    lib.eagle_attn_params_init(ctypes.byref(p))
    p.B, p.Tq, p.Tk, p.H, p.D, p.num_blocks = 1, 128, 128, 2, 128, 2
    p.scale = 128 ** -0.5
    fake = 1 << 20  # 16-byte aligned, never dereferenced: validation fails first
    p.q = p.cache_k = p.cache_v = p.out = p.lse = fake
    p.grad_out = p.dq = p.dk = p.dv = fake
    return p


@pytest.mark.parametrize("mutate,code", [
    (lambda p: setattr(p, "struct_size", 8), "EAGLE_ATTN_ERR_ABI"),
    (lambda p: setattr(p, "abi_version", 99), "EAGLE_ATTN_ERR_ABI"),
    (lambda p: setattr(p, "dtype", 7), "EAGLE_ATTN_ERR_DTYPE"),
    (lambda p: setattr(p, "D", 48), "EAGLE_ATTN_ERR_SHAPE"),
    (lambda p: setattr(p, "num_blocks", 0), "EAGLE_ATTN_ERR_SHAPE"),
    (lambda p: setattr(p, "Tk", 64), "EAGLE_ATTN_ERR_SHAPE"),          # NB > 1 needs Tk == Tq
    (lambda p: setattr(p, "q", None), "EAGLE_ATTN_ERR_NULL"),
    (lambda p: (setattr(p, "B", 2), setattr(p, "cu_seqlens", 1 << 20), setattr(p, "num_docs", 1)),
     "EAGLE_ATTN_ERR_VARLEN"),
    (lambda p: setattr(p, "q", (1 << 20) + 2), "EAGLE_ATTN_ERR_ALIGN"),
    (lambda p: setattr(p, "q_stride_t", 100), "EAGLE_ATTN_ERR_STRIDE"),
    (lambda p: setattr(p, "impl", 9), "EAGLE_ATTN_ERR_UNSUPPORTED"),
    (lambda p: (setattr(p, "q_tiles", 1 << 20), setattr(p, "num_q_tiles", -1)),
     "EAGLE_ATTN_ERR_SHAPE"),
    (lambda p: (setattr(p, "q_tiles", 1 << 20), setattr(p, "num_q_tiles", 1),
                setattr(p, "impl", 2)), "EAGLE_ATTN_ERR_UNSUPPORTED"),   # generic kernels
    (lambda p: setattr(p, "q_tile_rows", 1 << 20), "EAGLE_ATTN_ERR_SHAPE"),  # rows, no starts
])
def test_fwd_rejects_bad_arguments_on_host(mutate, code):
    p = _valid_params()
    mutate(p)
    rc = _lib.load().eagle_attn_fwd(ctypes.byref(p), None)
    assert _lib.STATUS[rc] == code


def test_bwd_rejects_missing_workspace():
    p = _valid_params()
    rc = _lib.load().eagle_attn_bwd(ctypes.byref(p), None)
    assert _lib.STATUS[rc] == "EAGLE_ATTN_ERR_WORKSPACE"


@pytest.mark.parametrize("mutate", [
    lambda p: setattr(p, "grad_mode", 2),                                # unknown mode
    lambda p: (setattr(p, "grad_mode", 1), setattr(p, "dtype", _lib.F32),
               setattr(p, "out_dtype", _lib.F32)),                       # fp32 inputs: no TC path
    lambda p: (setattr(p, "grad_mode", 1), setattr(p, "impl", 2)),       # generic kernels
    # query segments: the five-product kernel only
    lambda p: (setattr(p, "q_tiles", 1 << 20), setattr(p, "num_q_tiles", 1),
               setattr(p, "deterministic", 1)),
    lambda p: (setattr(p, "q_tiles", 1 << 20), setattr(p, "num_q_tiles", 1),
               setattr(p, "impl", 2)),
])
def test_bwd_rejects_unserved_grad_modes_on_host(mutate):
    p = _valid_params()
    mutate(p)
    rc = _lib.load().eagle_attn_bwd(ctypes.byref(p), None)
    assert _lib.STATUS[rc] == "EAGLE_ATTN_ERR_UNSUPPORTED"


def test_bwd_workspace_size_formula():
    p = _valid_params()
    n = _lib.load().eagle_attn_bwd_workspace_size(ctypes.byref(p))
    acc = 1 * 128 * 2 * 128 * 4
    dt = 1 * 2 * 128 * 4
    assert n == ((acc + 255) // 256) * 256 + ((dt + 255) // 256) * 256


def test_merge_rejects_bad_arguments_on_host():
    lib = _lib.load()
    f = 1 << 20
    assert _lib.STATUS[lib.attn_merge_out_lse(None, f, f, 0, f, 1, 1, 1, 128, 0, None)] == \
        "EAGLE_ATTN_ERR_NULL"
    assert _lib.STATUS[lib.attn_merge_out_lse(f, f, f, 5, f, 1, 1, 1, 128, 0, None)] == \
        "EAGLE_ATTN_ERR_DTYPE"
    assert _lib.STATUS[lib.attn_merge_out_lse(f, f, f, 0, f, 1, 1, 1, 96, 0, None)] == \
        "EAGLE_ATTN_ERR_SHAPE"
    assert _lib.STATUS[lib.attn_merge_out_lse(f + 4, f, f, 0, f, 1, 1, 1, 128, 0, None)] == \
        "EAGLE_ATTN_ERR_ALIGN"


def test_strerror_covers_every_status():
    lib = _lib.load()
    for code in _lib.STATUS:
        assert lib.eagle_attn_strerror(code).decode() != "unknown status"


def test_binding_error_type():
    with pytest.raises(ea.EagleAttnError):
        ea._check(-4, "x")


def test_finalize_alignment_rules_on_host():
    lib = _lib.load()
    f = 1 << 20
    assert _lib.STATUS[lib.attn_finalize(f + 2, f, _lib.F32, 8, None)] == "EAGLE_ATTN_ERR_ALIGN"
    assert _lib.STATUS[lib.attn_finalize(f, f + 1, _lib.BF16, 8, None)] == "EAGLE_ATTN_ERR_ALIGN"
    # element-aligned but not 16-byte aligned is served; count 0 launches nothing
    assert _lib.STATUS[lib.attn_finalize(f + 4, f + 4, _lib.F32, 0, None)] == "EAGLE_ATTN_OK"
    assert _lib.STATUS[lib.attn_finalize(f, None, _lib.F32, 8, None)] == "EAGLE_ATTN_ERR_NULL"


def test_empty_query_range_needs_no_buffers_on_host():
    """Tq == 0: nothing to compute, so the row buffers may be NULL and no
    kernel is launched (runs without a GPU)."""
    p = _valid_params()
    p.Tq, p.Tk, p.num_blocks = 0, 0, 2
    p.q = p.out = p.lse = p.cache_k = p.cache_v = None
    assert _lib.STATUS[_lib.load().eagle_attn_fwd(ctypes.byref(p), None)] == "EAGLE_ATTN_OK"
    p = _valid_params()
    p.Tq = 64
    p.Tk, p.num_blocks = 0, 1
    p.cache_k = p.cache_v = None  # no keys: allowed, the rows get lse = -inf
    p.q = None                    # but rows need their buffers
    assert _lib.STATUS[_lib.load().eagle_attn_fwd(ctypes.byref(p), None)] == "EAGLE_ATTN_ERR_NULL"
