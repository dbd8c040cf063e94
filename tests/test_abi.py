"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/*.h, and rejects bad arguments on the host."""
import ctypes
import glob
import os
import re

import pytest

from trainable_block_sparse_cube_b200 import build as vsa_build
from trainable_block_sparse_cube_b200 import vsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    vsa_build.build()
    return vsa.load()


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(vsa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "vsa_run" in names and "vsa_plan" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
    assert set(vsa.EXPORTED) == set(names)


def test_status_strings(lib):
    for code, name in vsa.STATUS.items():
        assert lib.vsa_status_string(code).decode() == name
    assert lib.vsa_status_string(99).decode() == "VSA_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(B=1, heads=2, T=8, H=8, W=8, D=64, topk=2, top_p=0.0, kmin=0, kmax=0)
    base.update(kw)
    return vsa.Config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(T=6), 2), (dict(W=10), 2), (dict(B=0), 2), (dict(heads=0), 2),
    (dict(D=96), 3), (dict(D=256), 3),
    (dict(topk=9), 1), (dict(topk=-1), 1),
    (dict(topk=0, top_p=0.0, kmin=1, kmax=4), 1), (dict(topk=0, top_p=1.5, kmin=1, kmax=4), 1),
    (dict(topk=0, top_p=0.9, kmin=5, kmax=4), 1), (dict(topk=0, top_p=0.9, kmin=0, kmax=4), 1),
    (dict(topk=0, top_p=0.9, kmin=1, kmax=9), 1),
    (dict(T=64, H=64, W=68), 3),    # C = 4352 > 4096
])
def test_invalid_configs(lib, kw, code):
    c = _cfg(**kw)
    assert lib.vsa_workspace_bytes(ctypes.byref(c)) == 0
    lay = vsa.WorkspaceLayout()
    assert lib.vsa_workspace_layout(ctypes.byref(c), ctypes.byref(lay)) == code
    h = ctypes.c_void_p()
    ws = ctypes.c_void_p(1 << 20)
    assert lib.vsa_plan(ctypes.byref(h), ctypes.byref(c), ws, 1 << 40) == code
    assert not h.value


def test_layout_sizes(lib):
    c = _cfg(B=2, heads=3, T=8, H=12, W=16, D=128, topk=5)
    lay = vsa.workspace_layout(c)
    BH, N, C, D = 6, 8 * 12 * 16, 8 * 12 * 16 // 64, 128
    assert lay.k_cube - lay.q_cube >= BH * N * D * 2
    assert lay.q_pool - lay.v_cube >= BH * N * D * 2
    assert lay.pool_split - lay.s_coarse >= BH * C * C * 4
    assert lay.total == lib.vsa_workspace_bytes(ctypes.byref(c))
    assert lay.p_split - lay.pool_split >= 9 * BH * C * D * 2
    assert lay.cnt - lay.p_split >= 3 * BH * C * ((C + 7) // 8 * 8) * 2
    assert lay.err - lay.order >= BH * C * 4
    offs = [lay.q_cube, lay.k_cube, lay.v_cube, lay.q_pool, lay.k_pool, lay.v_pool, lay.o_coarse, lay.s_coarse,
            lay.pool_split, lay.p_split, lay.cnt, lay.order, lay.err]
    assert offs == sorted(offs) and all(o % 1024 == 0 for o in offs)


def test_backward_workspace_size(lib):
    c = _cfg(B=1, heads=2, T=8, H=12, W=16, D=128, topk=5)
    BH, N, C, D = 2, 8 * 12 * 16, 8 * 12 * 16 // 64, 128
    nb = lib.vsa_backward_workspace_bytes(ctypes.byref(c))
    # at least: dO cube-major, statistics, dOc (+ terms), dS terms, pooled gradients, lists, orders
    assert nb >= BH * N * D * 2 + BH * C * 128 * 4 + BH * C * D * (4 + 6) + 3 * BH * C * ((C + 7) // 8 * 8) * 2
    assert lib.vsa_backward_workspace_bytes(ctypes.byref(_cfg(B=1, heads=2, T=6, H=12, W=16, D=128, topk=5))) == 0


def test_plan_argument_errors(lib):
    c = _cfg()
    h = ctypes.c_void_p()
    assert lib.vsa_plan(None, ctypes.byref(c), ctypes.c_void_p(1 << 20), 1 << 30) == 1
    assert lib.vsa_plan(ctypes.byref(h), ctypes.byref(c), None, 1 << 30) == 1
    assert lib.vsa_plan(ctypes.byref(h), ctypes.byref(c), ctypes.c_void_p((1 << 20) + 16), 1 << 30) == 4
    assert lib.vsa_plan(ctypes.byref(h), ctypes.byref(c), ctypes.c_void_p(1 << 20), 16) == 1
    assert lib.vsa_run(None, *([None] * 9)) == 1
    assert lib.vsa_run_host(None, *([None] * 9)) == 1
    assert lib.vsa_check(None) == 1
    assert lib.vsa_set_wait_limit_ns(None, 10 ** 9) == 1
    assert lib.vsa_set_debug_stall(None, 1) == 1
    assert lib.vsa_set_cube_major_copies(None, 1) == 1
    lib.vsa_plan_destroy(None)


def test_forward_rejects_bad_shape_without_touching_memory(lib):
    vp = ctypes.c_void_p
    code = lib.vsa_forward(vp(16), vp(16), vp(16), vp(16), vp(16), 1, 1, 6, 8, 8, 64, 2, ctypes.c_float(0.0),
                           vp(16), vp(16), None)
    assert code == 2
