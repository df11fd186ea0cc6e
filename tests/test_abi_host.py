"""Host-side tests of the C ABI (no GPU needed).

The library must load on a machine without a driver, export every function
include/arnq.h declares, and reject every illegal argument combination on the
host, before any CUDA call: the rejected calls below use fake, never
dereferenced device addresses, and each returns before the library would touch
a device.  Also checks the output-selection rules against the hand-written
truth table and against the oracle.
"""
import ctypes
import math

import pytest

import oracle
from int4_quant_b200 import _abi as A
from int4_quant_b200 import build as B
from tests._util import golden


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    A.lib()


def test_exports_every_header_symbol():
    names = A.header_functions()
    assert len(names) >= 8
    L = A.lib()
    for name in names:
        assert hasattr(L, name), name
    # and nothing of the oracle leaks into the product library
    assert not hasattr(L, "orc_add_rms_norm_dynamic_quant_v2")


def test_status_strings():
    for code in range(0, 12):
        s = A.arnq_status_string(code)
        assert s.startswith("ARNQ_")
    assert "unknown" in A.arnq_status_string(99)


def _mask(m):
    if m is None:
        return A.ARNQ_MASK_ABSENT
    return (1 if m[0] else 0) | (2 if m[1] else 0)


def test_selected_outputs_truth_table():
    t = golden("mask_truth_table.json")
    for mask, s1, s2, ok, y1, y2 in t["rows"]:
        st, on1, on2 = A.arnq_selected_outputs(_mask(mask), s1, s2)
        assert (st == A.ARNQ_OK) == ok, (mask, s1, s2)
        if ok:
            assert (on1, on2) == (y1, y2)
        else:
            assert st == A.ARNQ_ERR_MASK
        # the oracle reads the page the same way
        ost, o1, o2 = oracle.selected_outputs(None if mask is None else tuple(mask), s1, s2)
        assert (ost == oracle.ORC_OK) == ok and (not ok or (o1, o2) == (on1, on2))


def test_selected_outputs_rejects_unknown_mask_bits():
    assert A.arnq_selected_outputs(4, 0, 0)[0] == A.ARNQ_ERR_MASK
    assert A.arnq_selected_outputs(-2, 0, 0)[0] == A.ARNQ_ERR_MASK


def test_workspace_is_the_status_block_for_every_problem():
    # the per-row bookkeeping stays on chip: the workspace is the 256-byte
    # status block whatever the shape, dtype, code type and outputs
    for rows in (1, 2, 64, 8192, 16384, 2 ** 31 - 1):
        for n in (2, 8, 1000, 4096, 7168, 16384, A.ARNQ_MAX_N):
            for qdt in (A.ARNQ_INT8, A.ARNQ_INT4):
                for mask, s1, s2 in ((-1, 0, 0), (1, 1, 0), (3, 1, 1), (-1, 1, 1)):
                    st, nb = A.arnq_workspace_size(rows, n, A.ARNQ_BF16, qdt, mask, s1, s2)
                    assert st == A.ARNQ_OK and nb == A.ARNQ_WORKSPACE_BYTES, (rows, n, qdt, mask)


def test_workspace_size():
    st, nb = A.arnq_workspace_size(8192, 4096, A.ARNQ_BF16, A.ARNQ_INT8, 1, 1, 0)
    assert st == A.ARNQ_OK and nb == 256
    assert A.arnq_workspace_size(0, 4096, 0, 0, -1, 0, 0)[0] == A.ARNQ_ERR_EMPTY
    assert A.arnq_workspace_size(8, 0, 0, 0, -1, 0, 0)[0] == A.ARNQ_ERR_EMPTY
    assert A.arnq_workspace_size(8, 7, 0, A.ARNQ_INT4, -1, 0, 0)[0] == A.ARNQ_ERR_SHAPE
    assert A.arnq_workspace_size(8, A.ARNQ_MAX_N + 8, 0, 0, -1, 0, 0)[0] == A.ARNQ_ERR_SHAPE
    assert A.arnq_workspace_size(8, 64, 2, 0, -1, 0, 0)[0] == A.ARNQ_ERR_DTYPE
    assert A.arnq_workspace_size(8, 64, 0, 3, -1, 0, 0)[0] == A.ARNQ_ERR_DTYPE
    assert A.arnq_workspace_size(8, 60, 0, A.ARNQ_INT4_INT32, -1, 0, 0)[0] == A.ARNQ_ERR_SHAPE
    assert A.arnq_workspace_size(8, 64, 0, 0, 0, 0, 0)[0] == A.ARNQ_ERR_MASK
    assert A.arnq_workspace_size(-1, 64, 0, 0, -1, 0, 0)[0] == A.ARNQ_ERR_SHAPE
    L = A.lib()
    assert L.arnq_workspace_size(8, 64, 0, 0, -1, 0, 0, None) == A.ARNQ_ERR_NULL_PTR


# fake device addresses: 256-byte aligned, never dereferenced on the host
P = {k: 0x7F0000000000 + i * 0x100000 for i, k in enumerate(
    ["x1", "x2", "g", "b", "s1", "s2", "y1", "sc1", "y2", "sc2", "xo", "ws"])}


def run(**kw):
    a = dict(x1=P["x1"], x2=P["x2"], gamma=P["g"], beta=None, smooth1=None, smooth2=None,
             rows=16, n=64, dt=A.ARNQ_BF16, eps=1e-6, out_mask=A.ARNQ_MASK_ABSENT,
             qdt=A.ARNQ_INT8, y1=P["y1"], scale1=P["sc1"], y2=None, scale2=None, x_out=P["xo"],
             workspace=P["ws"], workspace_bytes=1 << 20, stream=None)
    a.update(kw)
    return A.arnq_run(**a)


@pytest.mark.parametrize("kw,expect", [
    (dict(x1=None), A.ARNQ_ERR_NULL_PTR),
    (dict(x2=None), A.ARNQ_ERR_NULL_PTR),
    (dict(gamma=None), A.ARNQ_ERR_NULL_PTR),
    (dict(y1=None), A.ARNQ_ERR_NULL_PTR),
    (dict(scale1=None), A.ARNQ_ERR_NULL_PTR),
    (dict(smooth1=P["s1"], smooth2=P["s2"], y2=None, scale2=P["sc2"]), A.ARNQ_ERR_NULL_PTR),
    (dict(out_mask=3, y2=P["y2"], scale2=None), A.ARNQ_ERR_NULL_PTR),
    (dict(rows=0), A.ARNQ_ERR_EMPTY),
    (dict(n=0), A.ARNQ_ERR_EMPTY),
    (dict(rows=-3), A.ARNQ_ERR_SHAPE),
    (dict(n=A.ARNQ_MAX_N + 2), A.ARNQ_ERR_SHAPE),
    (dict(n=63, qdt=A.ARNQ_INT4), A.ARNQ_ERR_SHAPE),
    (dict(n=60, qdt=A.ARNQ_INT4_INT32), A.ARNQ_ERR_SHAPE),
    (dict(qdt=A.ARNQ_INT4_INT32, y1=P["y1"] + 2), A.ARNQ_ERR_ALIGN),
    (dict(dt=5), A.ARNQ_ERR_DTYPE),
    (dict(qdt=-1), A.ARNQ_ERR_DTYPE),
    (dict(qdt=3), A.ARNQ_ERR_DTYPE),
    (dict(eps=-1e-6), A.ARNQ_ERR_EPS),
    (dict(eps=math.nan), A.ARNQ_ERR_EPS),
    (dict(eps=math.inf), A.ARNQ_ERR_EPS),
    # Constraints-section rules
    (dict(out_mask=2, smooth1=P["s1"], y2=P["y2"], scale2=P["sc2"]), A.ARNQ_ERR_MASK),
    (dict(out_mask=1, smooth2=P["s2"]), A.ARNQ_ERR_MASK),
    (dict(out_mask=0), A.ARNQ_ERR_MASK),
    (dict(smooth2=P["s2"]), A.ARNQ_ERR_MASK),
    (dict(out_mask=7), A.ARNQ_ERR_MASK),
    # alignment and workspace
    (dict(x1=P["x1"] + 1), A.ARNQ_ERR_ALIGN),
    (dict(gamma=P["g"] + 3), A.ARNQ_ERR_ALIGN),
    (dict(x_out=P["xo"] + 1), A.ARNQ_ERR_ALIGN),
    (dict(scale1=P["sc1"] + 2), A.ARNQ_ERR_ALIGN),
    (dict(workspace=None), A.ARNQ_ERR_WORKSPACE),
    (dict(workspace_bytes=8), A.ARNQ_ERR_WORKSPACE),
    (dict(workspace=P["ws"] + 4), A.ARNQ_ERR_ALIGN),
])
def test_run_rejects_on_the_host(kw, expect):
    assert run(**kw) == expect


def test_unselected_outputs_may_be_null():
    # mask [False, True] with no smooth scale: y1/scale1 unused, so NULL is no
    # error; the call is then rejected for the missing y2 (proving it got past
    # the y1 checks without touching a device).
    assert run(out_mask=2, y1=None, scale1=None, y2=None, scale2=None) == A.ARNQ_ERR_NULL_PTR


def test_v1_and_no_add_entry_points_validate():
    L = A.lib()
    assert A.arnq_run_v1(P["x1"], P["x2"], None, None, None, 8, 64, 0, 1e-6, 0, P["y1"],
                         P["sc1"], None, None, P["xo"], P["ws"], 256, None) == A.ARNQ_ERR_NULL_PTR
    assert A.arnq_run_v1(P["x1"], P["x2"], P["g"], None, P["s2"], 8, 64, 0, 1e-6, 0, P["y1"],
                         P["sc1"], None, None, P["xo"], P["ws"], 256, None) == A.ARNQ_ERR_MASK
    assert A.arnq_rms_norm_dynamic_quant(P["x1"], P["g"], None, None, 0, 64, 0, 1e-6, 0,
                                         P["y1"], P["sc1"], P["ws"], 256, None) == A.ARNQ_ERR_EMPTY
    assert A.arnq_rms_norm_dynamic_quant(P["x1"], P["g"], None, None, 8, 64, 0, 1e-6, 0,
                                         None, P["sc1"], P["ws"], 256, None) == A.ARNQ_ERR_NULL_PTR
    assert L.arnq_run_planned(None, None, None, None, None, None, 1, 8, 0, 0.0, -1, 0, None,
                              None, None, None, None, None, 0, None, None) == A.ARNQ_ERR_NULL_PTR


def test_plan_struct_layout():
    assert ctypes.sizeof(A.arnq_plan) == 44
    assert ctypes.sizeof(A.arnq_workspace_status) == 16


def test_static_scratch_entry_validates_on_the_host():
    # rejected before the library touches a device (no set-up, no copy)
    assert A.arnq_run_static_scratch(None, None, None, None, None, None, 8, 64, 0, 1e-6, -1, 0,
                                     None, None, None, None, None, None) == A.ARNQ_ERR_NULL_PTR
    assert A.arnq_run_static_scratch(P["x1"], P["x2"], P["g"], None, None, None, 0, 64, 0, 1e-6,
                                     -1, 0, P["y1"], P["sc1"], None, None, None,
                                     None) == A.ARNQ_ERR_EMPTY
    assert A.arnq_run_static_scratch(P["x1"], P["x2"], P["g"], None, None, P["s2"], 8, 64, 0, 1e-6,
                                     -1, 0, P["y1"], P["sc1"], None, None, None,
                                     None) == A.ARNQ_ERR_MASK
    # the static array covers the workspace of every valid problem, the largest too
    assert A.ARNQ_STATIC_SCRATCH_BYTES >= A.arnq_workspace_size(2 ** 31 - 1, A.ARNQ_MAX_N, 0, 1,
                                                                 3, 1, 1)[1]


@pytest.mark.parametrize("field,value", [
    ("early_params", 2), ("early_params", -1), ("test_hold_bytes", 65537), ("test_hold_bytes", -16),
    ("wait_limit_us", -1), ("grid", -2), ("stages", -1), ("cluster", -4)])
def test_plan_fields_out_of_range_are_refused_on_the_host(field, value):
    p = A.arnq_plan()
    setattr(p, field, value)
    st = A.arnq_run_planned(P["x1"], P["x2"], P["g"], None, None, None, 16, 64, A.ARNQ_BF16, 1e-6,
                            A.ARNQ_MASK_ABSENT, A.ARNQ_INT8, P["y1"], P["sc1"], None, None,
                            P["xo"], P["ws"], 256, None, p)
    assert st == A.ARNQ_ERR_PLAN
