"""The no-allocation entry point arnq_run_static_scratch on a GPU.

Its scratch is a file-scope device array inside the library; this checks that
two calls in a row each give exactly what arnq_run (caller workspace) gives on
the same inputs and plan, for INT8 with two outputs and for packed INT4.  The
file name sorts last so the suite also runs it after every other GPU test.
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


@pytest.mark.parametrize("case", ["int8_two_outputs", "int4_fp16"])
def test_static_scratch_equals_workspace_entry_on_two_calls(case):
    if case == "int8_two_outputs":
        w = wl.random_case(300, 4096, seed=41, beta=True, smooth1=True, smooth2=True,
                           mask=(True, True))
        mask, on2 = A.ARNQ_MASK_Y1 | A.ARNQ_MASK_Y2, True
    else:
        w = wl.random_case(257, 5120, dtype="fp16", qdtype="int4", seed=42, beta=True)
        mask, on2 = A.ARNQ_MASK_ABSENT, False
    ins = dict(x1=_dev(w.x1, w.dtype), x2=_dev(w.x2, w.dtype), g=_dev(w.gamma, w.dtype),
               b=_dev(w.beta, w.dtype), s1=_dev(w.smooth1, w.dtype), s2=_dev(w.smooth2, w.dtype))
    ref = _outputs(w, on2)
    _call("ws", w, ins, ref, mask)
    for _ in range(2):  # two calls in a row through the static scratch
        got = _outputs(w, on2)
        _call("static", w, ins, got, mask)
        for k in ("y1", "s1", "y2", "s2", "xo"):
            if ref[k] is None:
                continue
            assert torch.equal(got[k].view(torch.uint8), ref[k].view(torch.uint8)), k


def test_static_scratch_rejects_on_the_host_first():
    # a rejected call returns before any device work (and before set-up)
    assert A.arnq_run_static_scratch(None, None, None, None, None, None, 8, 64, 0, 1e-6, -1, 0,
                                     None, None, None, None, None, None) == A.ARNQ_ERR_NULL_PTR
