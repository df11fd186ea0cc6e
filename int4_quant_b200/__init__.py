"""B200 (sm_100a) fused residual add + RMSNorm + per-row dynamic quantization.

The operator of the CANN page "aclnnAddRmsNormDynamicQuantV2" (and its
no-add sibling "aclnnRmsNormDynamicQuant"), computed by the hand-written
kernels of ``libarnq.so`` behind the C ABI in ``include/arnq.h``.

``int4_quant_b200._abi`` is the ctypes binding (same names as the C entry
points).  The functions below are the torch-facing calls: they allocate the
outputs with torch and hand raw pointers to the library; every step of the
operator runs in the library's kernels.
"""
from __future__ import annotations

from typing import Optional, Tuple

from . import _abi
from ._abi import ArnqError  # noqa: F401

_DT = {"torch.bfloat16": _abi.ARNQ_BF16, "torch.float16": _abi.ARNQ_FP16}
_QDT = {"int8": _abi.ARNQ_INT8, "int4": _abi.ARNQ_INT4, "int4_int32": _abi.ARNQ_INT4_INT32}


def _codes_like(lead, n, qdtype):
    """(shape, torch dtype) of a quantized output: int8 [..., n], packed uint8
    [..., n/2], or int32 [..., n/8] words of eight INT4 codes."""
    import torch
    if qdtype == "int8":
        return lead + (n,), torch.int8
    if qdtype == "int4_int32":
        return lead + (n // 8,), torch.int32
    if qdtype == "int4":
        return lead + (n // 2,), torch.uint8
    raise ValueError(f"unknown qdtype {qdtype!r}")
_workspaces = {}


def mask_code(output_mask) -> int:
    """None -> absent; (m0, m1) -> bit 0 = m0 (y1), bit 1 = m1 (y2)."""
    if output_mask is None:
        return _abi.ARNQ_MASK_ABSENT
    m0, m1 = output_mask
    return (_abi.ARNQ_MASK_Y1 if m0 else 0) | (_abi.ARNQ_MASK_Y2 if m1 else 0)


def workspace(device, nbytes: int, stream=None):
    """A device workspace of at least nbytes with a zeroed status block, cached
    per (device, stream) and grown on demand: calls on one stream may share it,
    calls that overlap on other streams get their own."""
    import torch
    key = (str(device), _abi._stream(stream) or 0)
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def workspace_status(ws) -> Tuple[int, int]:
    """(code, row) of a workspace's status block (synchronizes on its stream)."""
    import torch
    host = ws[:16].cpu().numpy().view("int32")
    return int(host[0]), int(host[2:4].view("int64")[0])


def _check(t, name, dtype=None):
    import torch
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")


def add_rms_norm_dynamic_quant(x1, x2, gamma, beta=None, smooth1=None, smooth2=None, *,
                               eps: float = 1e-6, output_mask=None, qdtype: str = "int8",
                               stream=None, out: Optional[dict] = None,
                               constant_params: bool = False):
    """aclnnAddRmsNormDynamicQuantV2 on CUDA tensors.

    x1, x2: [..., n] bf16 or fp16; gamma, beta, smooth1, smooth2: [n] same dtype.
    Returns (y1, scale1, y2, scale2, x_out); an output that is not selected is
    None.  y is int8 [..., n]; for qdtype="int4", uint8 [..., n/2] holding
    two codes per byte (even column in the low nibble); for
    qdtype="int4_int32", int32 [..., n/8] holding eight codes per word (column
    8w + k in bits 4k..4k+3).  `out` may pass preallocated tensors under the
    same keys.  constant_params=True promises that the work queued before
    this call on the stream does not write gamma, beta or the smooth scales
    (weights, as in inference): the kernel then loads them before it waits
    for that work (the plan's early_params).
    """
    import torch
    _check(x1, "x1")
    dt = x1.dtype
    for name, t in (("x2", x2), ("gamma", gamma), ("beta", beta), ("smooth1", smooth1),
                    ("smooth2", smooth2)):
        _check(t, name, dt)
    if str(dt) not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    n = x1.shape[-1]
    rows = x1.numel() // n if n else 0
    mc = mask_code(output_mask)
    st, on1, on2 = _abi.arnq_selected_outputs(mc, smooth1 is not None, smooth2 is not None)
    if st != _abi.ARNQ_OK:
        raise ArnqError(st, "arnq_selected_outputs")
    lead = tuple(x1.shape[:-1])
    cshape, cdt = _codes_like(lead, n, qdtype)
    out = dict(out or {})

    def alloc(key, shape, dtype, on):
        if not on:
            return None
        if key not in out or out[key] is None:
            out[key] = torch.empty(shape, dtype=dtype, device=x1.device)
        return out[key]

    y1 = alloc("y1", cshape, cdt, on1)
    s1 = alloc("scale1", lead, torch.float32, on1)
    y2 = alloc("y2", cshape, cdt, on2)
    s2 = alloc("scale2", lead, torch.float32, on2)
    xo = alloc("x_out", tuple(x1.shape), dt, True)
    st, nbytes = _abi.arnq_workspace_size(rows, n, _DT[str(dt)], _QDT[qdtype], mc,
                                          smooth1 is not None, smooth2 is not None)
    if st != _abi.ARNQ_OK:
        raise ArnqError(st, "arnq_workspace_size")
    if stream is None:
        stream = torch.cuda.current_stream(x1.device)
    ws = workspace(x1.device, nbytes, stream)
    args = (x1, x2, gamma, beta, smooth1, smooth2, rows, n, _DT[str(dt)], eps, mc, _QDT[qdtype],
            y1, s1, y2, s2, xo, ws, ws.numel(), stream)
    if constant_params:
        plan = _abi.arnq_plan()
        plan.early_params = 1
        st = _abi.arnq_run_planned(*args, plan)
    else:
        st = _abi.arnq_run(*args)
    if st != _abi.ARNQ_OK:
        raise ArnqError(st, "arnq_run")
    return y1, s1, y2, s2, xo


def rms_norm_dynamic_quant(x, gamma, beta=None, smooth=None, *, eps: float = 1e-6,
                           qdtype: str = "int8", stream=None):
    """aclnnRmsNormDynamicQuant on CUDA tensors: returns (y, scale)."""
    import torch
    _check(x, "x")
    dt = x.dtype
    for name, t in (("gamma", gamma), ("beta", beta), ("smooth", smooth)):
        _check(t, name, dt)
    if str(dt) not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    n = x.shape[-1]
    rows = x.numel() // n if n else 0
    lead = tuple(x.shape[:-1])
    cshape, cdt = _codes_like(lead, n, qdtype)
    y = torch.empty(cshape, dtype=cdt, device=x.device)
    scale = torch.empty(lead, dtype=torch.float32, device=x.device)
    st, nbytes = _abi.arnq_workspace_size(rows, n, _DT[str(dt)], _QDT[qdtype],
                                          _abi.ARNQ_MASK_ABSENT, smooth is not None, False)
    if st != _abi.ARNQ_OK:
        raise ArnqError(st, "arnq_workspace_size")
    if stream is None:
        stream = torch.cuda.current_stream(x.device)
    ws = workspace(x.device, nbytes, stream)
    st = _abi.arnq_rms_norm_dynamic_quant(x, gamma, beta, smooth, rows, n, _DT[str(dt)], eps,
                                          _QDT[qdtype], y, scale, ws, ws.numel(), stream)
    if st != _abi.ARNQ_OK:
        raise ArnqError(st, "arnq_rms_norm_dynamic_quant")
    return y, scale
