"""The no-allocation entry point arnq_run_static_scratch on a GPU.

It serves callers that cannot allocate device memory at the point of the
call; its scratch (the status block) is a file-scope device array inside
the library.  These tests check that two calls in a row each give exactly
what arnq_run with a caller workspace gives on the same inputs and plan:
INT8 with two outputs, packed INT4, rows shared by a thread-block cluster,
and a large row count.
The file name sorts last so that a run stopping at the first failure has run
every other GPU test first; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from int4_quant_b200 import _abi as A
from int4_quant_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _dev(bits, dtype):
    if bits is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()
    return t.view(torch.bfloat16 if dtype == "bf16" else torch.float16)


def _outputs(w, on2):
    cb = w.n if w.qdtype == "int8" else w.n // 2
    mk = lambda: torch.full((w.rows, cb), 0x5A, dtype=torch.uint8, device="cuda")  # canary
    sc = lambda: torch.full((w.rows,), -1.0, dtype=torch.float32, device="cuda")
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    return dict(y1=mk(), s1=sc(), y2=mk() if on2 else None, s2=sc() if on2 else None,
                xo=torch.empty((w.rows, w.n), dtype=tdt, device="cuda"))


def _call(entry, w, ins, out, mask):
    dt = A.ARNQ_BF16 if w.dtype == "bf16" else A.ARNQ_FP16
    qd = A.ARNQ_INT8 if w.qdtype == "int8" else A.ARNQ_INT4
    args = [ins["x1"], ins["x2"], ins["g"], ins["b"], ins["s1"], ins["s2"], w.rows, w.n, dt, w.eps,
            mask, qd, out["y1"], out["s1"], out["y2"], out["s2"], out["xo"]]
    if entry == "ws":
        nb = A.arnq_workspace_size(w.rows, w.n, dt, qd, mask, ins["s1"] is not None,
                                   ins["s2"] is not None)[1]
        ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
        st = A.arnq_run(*args, ws, nb, torch.cuda.current_stream())
    else:
        st = A.arnq_run_static_scratch(*args, torch.cuda.current_stream())
    assert st == A.ARNQ_OK, A.arnq_status_string(st)
    torch.cuda.synchronize()


def _case(name):
    if name == "int8_two_outputs":
        w = wl.random_case(300, 4096, seed=41, beta=True, smooth1=True, smooth2=True,
                           mask=(True, True))
        return w, A.ARNQ_MASK_Y1 | A.ARNQ_MASK_Y2, True
    if name == "int4_fp16":
        return wl.random_case(257, 5120, dtype="fp16", qdtype="int4", seed=42, beta=True), \
            A.ARNQ_MASK_ABSENT, False
    if name == "dual_16384":   # a cluster shares each row
        w = wl.random_case(16, 16384, seed=43, beta=True, smooth1=True, smooth2=True,
                           mask=(True, True))
        return w, A.ARNQ_MASK_Y1 | A.ARNQ_MASK_Y2, True
    if name.startswith("rows_16384_"):   # cluster plans, one row per cluster
        rows = int(name.rsplit("_", 1)[1])
        return wl.random_case(rows, 16384, seed=44 + rows, beta=True, smooth1=True), \
            A.ARNQ_MASK_ABSENT, False
    if name == "rows_2048x4096":   # several rows per CTA
        return wl.random_case(2048, 4096, seed=45, x_sigma=(1.0, 0.5), beta=True, smooth1=True,
                              mask=(True, False)), A.ARNQ_MASK_Y1, False
    raise KeyError(name)


def _inputs(w):
    return dict(x1=_dev(w.x1, w.dtype), x2=_dev(w.x2, w.dtype), g=_dev(w.gamma, w.dtype),
                b=_dev(w.beta, w.dtype), s1=_dev(w.smooth1, w.dtype), s2=_dev(w.smooth2, w.dtype))


def _same(got, ref):
    for k in ("y1", "s1", "y2", "s2", "xo"):
        if ref[k] is None:
            continue
        assert torch.equal(got[k].view(torch.uint8), ref[k].view(torch.uint8)), k


# Each case: the no-allocation entry point, twice in a row, against arnq_run
# with a caller workspace (same inputs, same plan: identical bits).  The
# cluster cases run right after a dual-output 16384-column call through the
# same array, and the last case right after the others, so each starts from
# whatever the previous calls left in the array.
CASES = ["int8_two_outputs", "int4_fp16", "dual_16384", "rows_16384_8", "rows_16384_128",
         "rows_2048x4096"]


@pytest.mark.parametrize("case", CASES)
def test_static_scratch_equals_workspace_entry_on_two_calls(case):
    w, mask, on2 = _case(case)
    ins = _inputs(w)
    ref = _outputs(w, on2)
    _call("ws", w, ins, ref, mask)
    if case.startswith("rows_16384_"):
        # leave a dual-output cluster call's traces in the array first
        wd, maskd, _ = _case("dual_16384")
        _call("static", wd, _inputs(wd), _outputs(wd, True), maskd)
    for _ in range(2):  # two calls in a row through the static scratch
        got = _outputs(w, on2)
        _call("static", w, ins, got, mask)
        _same(got, ref)


def test_static_scratch_sequence_in_one_process():
    # the whole sequence again, back to back, with no test in between
    results = {}
    for case in CASES:
        w, mask, on2 = _case(case)
        ins = _inputs(w)
        ref = _outputs(w, on2)
        _call("ws", w, ins, ref, mask)
        got = _outputs(w, on2)
        _call("static", w, ins, got, mask)
        _same(got, ref)
        results[case] = True
    assert all(results.values())


def test_static_scratch_rejects_on_the_host_first():
    # a rejected call returns before any device work (and before set-up)
    assert A.arnq_run_static_scratch(None, None, None, None, None, None, 8, 64, 0, 1e-6, -1, 0,
                                     None, None, None, None, None, None) == A.ARNQ_ERR_NULL_PTR
