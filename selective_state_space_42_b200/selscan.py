"""Python binding of libselscan (include/selscan.h): argument marshalling only.

Every function here checks that the tensors it is handed are what the C ABI
expects (device, dtype, contiguity, shape) and passes raw pointers, sizes and
the current CUDA stream to the library. All computation runs in the CUDA
kernels behind the ABI. If the shared library is missing, every call raises
(``SelscanUnavailable``); there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libselscan.so")

SELSCAN_F32 = 0
SELSCAN_BF16 = 1
SELSCAN_MAX_DSTATE = 256
SELSCAN_MAX_DSTATE_BWD = 256

STATUS = {
    0: "SELSCAN_OK", -1: "SELSCAN_ERR_NULL_ARG", -2: "SELSCAN_ERR_BAD_DIM",
    -3: "SELSCAN_ERR_BAD_DTYPE", -4: "SELSCAN_ERR_MISALIGNED",
    -5: "SELSCAN_ERR_DSTATE_UNSUPPORTED", -6: "SELSCAN_ERR_CUDA",
    -7: "SELSCAN_ERR_ALIAS", -8: "SELSCAN_ERR_WORKSPACE",
}

# bytes of the fixed workspace array behind selscan_fwd_noalloc
SELSCAN_NOALLOC_WORKSPACE_BYTES = 16 << 20

_vp = ctypes.c_void_p


class FwdOptions(ctypes.Structure):
    """selscan_fwd_options_t (include/selscan.h)."""
    _fields_ = [("initial_state", ctypes.c_void_p), ("conv_weight", ctypes.c_void_p),
                ("conv_bias", ctypes.c_void_p), ("conv_init", ctypes.c_void_p),
                ("conv_width", ctypes.c_int), ("bbar_mode", ctypes.c_int)]


class StepOptions(ctypes.Structure):
    """selscan_step_options_t (include/selscan.h)."""
    _fields_ = [("conv_state", ctypes.c_void_p), ("conv_weight", ctypes.c_void_p),
                ("conv_bias", ctypes.c_void_p), ("conv_width", ctypes.c_int),
                ("bbar_mode", ctypes.c_int)]


class BwdOptions(ctypes.Structure):
    """selscan_bwd_options_t (include/selscan.h)."""
    _fields_ = [("initial_state", ctypes.c_void_p), ("dinitial_state", ctypes.c_void_p),
                ("conv_weight", ctypes.c_void_p), ("conv_bias", ctypes.c_void_p),
                ("conv_width", ctypes.c_int), ("dconv_weight", ctypes.c_void_p),
                ("dconv_bias", ctypes.c_void_p), ("bbar_mode", ctypes.c_int)]


BBAR_MODES = {"delta": 0, "zoh": 1}
_i64 = ctypes.c_int64
_int = ctypes.c_int

# name -> (restype, argtypes), mirroring include/selscan.h
SIGNATURES = {
    "selscan_fwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp, _vp,
                           _i64, _i64, _i64, _i64, _int, _vp]),
    "selscan_state_update": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                    _int, _vp, _i64, _i64, _i64, _int, _vp]),
    "selscan_fwd_from_state": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                      _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp]),
    "selscan_fwd_conv": (_int, [_vp, _vp, _vp, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _int, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp]),
    "selscan_fwd_noalloc": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _vp,
                                   _vp, _i64, _i64, _i64, _i64, _int, _vp]),
    "selscan_fwd_plan": (_int, [_i64, _i64, _i64, _i64, ctypes.POINTER(_i64),
                                ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "selscan_bwd": (_int, [_vp] * 8 + [_int] + [_vp] * 10
                    + [_i64, _i64, _i64, _i64, _int, _vp]),
    "selscan_bwd_workspace_bytes": (_i64, [_i64, _i64, _i64, _i64]),
    "selscan_bwd_conv": (_int, [_vp, _vp, _vp, _int] + [_vp] * 7 + [_int] + [_vp] * 14
                         + [_i64, _i64, _i64, _i64, _int, _vp, _i64, _vp]),
    "selscan_bwd_conv_workspace_bytes": (_i64, [_i64, _i64, _i64, _i64]),
    "selscan_bwd_ex": (_int, [_vp] * 8 + [_int, _vp, _vp, ctypes.POINTER(BwdOptions)]
                       + [_vp] * 8 + [_i64, _i64, _i64, _i64, _int, _vp, _i64, _vp]),
    "selscan_bwd_from_state": (_int, [_vp] * 8 + [_int] + [_vp] * 12
                               + [_i64, _i64, _i64, _i64, _int, _vp, _i64, _vp]),
    "selscan_bwd_workspace": (_int, [_vp] * 8 + [_int] + [_vp] * 10
                              + [_i64, _i64, _i64, _i64, _int, _vp, _i64, _vp]),
    "selscan_state_update_conv": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _vp, _vp, _vp, _vp,
                                         _vp, _vp, _vp, _int, _vp, _i64, _i64, _i64, _int,
                                         _vp]),
    "selscan_fwd_ex": (_int, [_vp] * 8 + [_int, ctypes.POINTER(FwdOptions), _vp, _vp, _i64,
                                          _i64, _i64, _i64, _int, _vp]),
    "selscan_state_update_ex": (_int, [_vp] * 9 + [_int, ctypes.POINTER(StepOptions), _vp,
                                                   _i64, _i64, _i64, _int, _vp]),
    "selscan_ssd_fwd": (_int, [_vp] * 8 + [_int, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                          _int, _vp, _i64, _vp]),
    "selscan_ssd_workspace_bytes": (_i64, [_i64, _i64, _i64, _i64, _i64]),
    "selscan_device_status": (_int, [ctypes.POINTER(_int), _int]),
    "selscan_status_string": (ctypes.c_char_p, [_int]),
    "selscan_last_cuda_error": (ctypes.c_char_p, []),
}


class SelscanUnavailable(RuntimeError):
    """libselscan.so is not built or cannot be loaded."""


class SelscanError(RuntimeError):
    def __init__(self, status: int, detail: str = ""):
        self.status = status
        msg = f"{STATUS.get(status, status)}: {detail}"
        super().__init__(msg)


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the shared library; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise SelscanUnavailable(
            f"{path} is missing: build it with `python -m "
            f"selective_state_space_42_b200.build` (nvcc, sm_100a)")
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:
        raise SelscanUnavailable(f"cannot load {path}: {e}") from e
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def selscan_status_string(status: int) -> str:
    return load_library().selscan_status_string(int(status)).decode()


def selscan_last_cuda_error() -> str:
    return load_library().selscan_last_cuda_error().decode()


def _check(status: int):
    if status != 0:
        detail = selscan_status_string(status)
        if status == -6:
            detail += f" ({selscan_last_cuda_error()})"
        raise SelscanError(status, detail)


# ---- tensor marshalling ----------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return SELSCAN_F32
    if t.dtype == torch.bfloat16:
        return SELSCAN_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t, name, shape=None, dtype=None, device=None, required=True):
    if t is None:
        if required:
            raise ValueError(f"{name} is required")
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream_ptr(stream, device):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def selscan_fwd_plan(batch: int, seqlen: int, dim: int, dstate: int) -> dict:
    """Launch plan of selscan_fwd for these sizes (C ABI ``selscan_fwd_plan``):
    {"chunks", "launches", "workspace_bytes"}."""
    c, n, w = _i64(), _i64(), _i64()
    _check(load_library().selscan_fwd_plan(batch, seqlen, dim, dstate, ctypes.byref(c),
                                           ctypes.byref(n), ctypes.byref(w)))
    return {"chunks": c.value, "launches": n.value, "workspace_bytes": w.value}


def selscan_device_status(clear: bool = False) -> int:
    """The library's sticky device-side error word on the current device (C
    ABI ``selscan_device_status``); 0 when no device wait has given up."""
    v = _int()
    _check(load_library().selscan_device_status(ctypes.byref(v), int(bool(clear))))
    return v.value


def selscan_fwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                y=None, final_state=None, return_final_state=False, stream=None,
                initial_state=None, conv_weight=None, conv_bias=None, conv_init=None,
                bbar="delta"):
    """Selective scan over whole sequences (C ABI ``selscan_fwd``;
    ``selscan_fwd_from_state`` when ``initial_state`` is given;
    ``selscan_fwd_conv`` when ``conv_weight`` is given).

    x, delta, z: [batch, L, dim]; B, C: [batch, L, dstate] (same dtype as x,
    float32 or bfloat16); A: [dim, dstate] float32; D, delta_bias: [dim]
    float32; initial_state: [batch, dim, dstate] float32 (the state before the
    first token; None: zero; may be the same tensor as final_state).
    conv_weight [dim, K] (K ≤ 4), conv_bias [dim], conv_init [batch, dim, 3]
    float32: x is then the input of the causal depthwise conv + SiLU in front
    of the scan. bbar: "delta" (Δ·B·x) or "zoh" (zero-order hold, C ABI
    ``selscan_fwd_ex``). Returns y (allocated if not given) or (y, final_state)."""
    if bbar != "delta":
        return _fwd("selscan_fwd_ex", x, delta, A, B, C, D, z, delta_bias, softplus, y,
                    final_state, return_final_state, stream, initial_state=initial_state,
                    conv=(conv_weight, conv_bias, conv_init), bbar=bbar)
    if conv_weight is not None:
        return _fwd("selscan_fwd_conv", x, delta, A, B, C, D, z, delta_bias, softplus, y,
                    final_state, return_final_state, stream, initial_state=initial_state,
                    conv=(conv_weight, conv_bias, conv_init))
    if initial_state is not None:
        return _fwd("selscan_fwd_from_state", x, delta, A, B, C, D, z, delta_bias, softplus,
                    y, final_state, return_final_state, stream, initial_state=initial_state)
    return _fwd("selscan_fwd", x, delta, A, B, C, D, z, delta_bias, softplus, y,
                final_state, return_final_state, stream)


def selscan_fwd_noalloc(x, delta, A, B, C, D=None, z=None, delta_bias=None,
                        softplus=True, y=None, final_state=None,
                        return_final_state=False, stream=None):
    """selscan_fwd whose chunk workspace is the library's fixed device array
    (C ABI ``selscan_fwd_noalloc``): the library allocates nothing. For
    callers that cannot allocate device memory, pass y (and final_state)
    preallocated; otherwise this wrapper allocates them with torch."""
    return _fwd("selscan_fwd_noalloc", x, delta, A, B, C, D, z, delta_bias, softplus,
                y, final_state, return_final_state, stream)


def _fwd(entry, x, delta, A, B, C, D, z, delta_bias, softplus, y, final_state,
         return_final_state, stream, initial_state=None, conv=None, bbar="delta"):
    torch = _torch()
    if x.dim() != 3:
        raise ValueError("x must be [batch, L, dim]")
    batch, L, dim = x.shape
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError("A must be [dim, dstate]")
    N = A.shape[1]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty(batch, dim, N, device=dev, dtype=torch.float32)
    f32 = torch.float32
    args = [_ptr(x, "x", (batch, L, dim), dt, dev)]
    if entry == "selscan_fwd_conv":
        cw, cbias, cinit = conv
        if cw.dim() != 2 or cw.shape[0] != dim:
            raise ValueError("conv_weight must be [dim, K]")
        args += [_ptr(cw, "conv_weight", (dim, cw.shape[1]), f32, dev),
                 _ptr(cbias, "conv_bias", (dim,), f32, dev, required=False),
                 int(cw.shape[1]),
                 _ptr(cinit, "conv_init", (batch, dim, 3), f32, dev, required=False)]
    args += [
        _ptr(delta, "delta", (batch, L, dim), dt, dev),
        _ptr(A, "A", (dim, N), f32, dev),
        _ptr(B, "B", (batch, L, N), dt, dev),
        _ptr(C, "C", (batch, L, N), dt, dev),
        _ptr(D, "D", (dim,), f32, dev, required=False),
        _ptr(z, "z", (batch, L, dim), dt, dev, required=False),
        _ptr(delta_bias, "delta_bias", (dim,), f32, dev, required=False),
        int(bool(softplus)),
    ]
    keep = []  # objects the C call points into
    if entry == "selscan_fwd_ex":
        cw, cbias, cinit = conv
        if bbar not in BBAR_MODES:
            raise ValueError(f"bbar must be one of {list(BBAR_MODES)}")
        opts = FwdOptions(
            _ptr(initial_state, "initial_state", (batch, dim, N), f32, dev, required=False),
            None if cw is None else _ptr(cw, "conv_weight", (dim, cw.shape[1]), f32, dev),
            None if cw is None else _ptr(cbias, "conv_bias", (dim,), f32, dev, required=False),
            None if cw is None else _ptr(cinit, "conv_init", (batch, dim, 3), f32, dev,
                                         required=False),
            0 if cw is None else int(cw.shape[1]), BBAR_MODES[bbar])
        keep.append(opts)
        args.append(ctypes.byref(opts))
    if entry == "selscan_fwd_from_state":
        args.append(_ptr(initial_state, "initial_state", (batch, dim, N), f32, dev))
    elif entry == "selscan_fwd_conv":
        args.append(_ptr(initial_state, "initial_state", (batch, dim, N), f32, dev,
                         required=False))
    args += [
        _ptr(y, "y", (batch, L, dim), dt, dev),
        _ptr(final_state, "final_state", (batch, dim, N), f32, dev, required=False),
        batch, L, dim, N, code, _stream_ptr(stream, dev),
    ]
    _check(getattr(load_library(), entry)(*args))
    if return_final_state:
        return y, final_state
    return y


def selscan_bwd(x, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                dy=None, dfinal_state=None, stream=None, allocate_in_library=False,
                initial_state=None, conv_weight=None, conv_bias=None, bbar="delta"):
    """Gradient of ``selscan_fwd`` for the loss Σ dy·y + Σ
    dfinal_state·final_state. Inputs as for ``selscan_fwd``; dy has y's shape
    and dtype, dfinal_state is [batch, dim, dstate] float32 or None. Returns a
    dict: dx, ddelta, dz (x's dtype; dz None without z), dA, dB, dC, dD,
    ddelta_bias (float32).

    The workspace comes from torch's caching allocator (C ABI
    ``selscan_bwd_workspace``); with ``allocate_in_library`` the library
    allocates it on the stream instead (C ABI ``selscan_bwd``). With
    ``initial_state`` (the forward's, [batch, dim, dstate] float32) the dict
    also holds its gradient ``dh0`` (C ABI ``selscan_bwd_from_state``). With
    ``conv_weight`` [dim, K] (and ``conv_bias``), x is the input of the causal
    conv + SiLU in front of the scan (C ABI ``selscan_bwd_conv``): dx is then
    the gradient w.r.t. that input, and the dict also holds ``dconv_weight``
    and ``dconv_bias``. ``bbar="zoh"`` differentiates the forward's ZOH input
    term (C ABI ``selscan_bwd_ex``, which takes all of these options)."""
    torch = _torch()
    if x.dim() != 3:
        raise ValueError("x must be [batch, L, dim]")
    batch, L, dim = x.shape
    if A.dim() != 2 or A.shape[0] != dim:
        raise ValueError("A must be [dim, dstate]")
    N = A.shape[1]
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    f32 = torch.float32
    out = dict(
        dx=torch.empty_like(x), ddelta=torch.empty_like(x),
        dz=torch.empty_like(x) if z is not None else None,
        dA=torch.empty(dim, N, device=dev, dtype=f32),
        dB=torch.empty(batch, L, N, device=dev, dtype=f32),
        dC=torch.empty(batch, L, N, device=dev, dtype=f32),
        dD=torch.empty(dim, device=dev, dtype=f32),
        ddelta_bias=torch.empty(dim, device=dev, dtype=f32))
    args = [
        _ptr(x, "x", (batch, L, dim), dt, dev),
        _ptr(delta, "delta", (batch, L, dim), dt, dev),
        _ptr(A, "A", (dim, N), f32, dev),
        _ptr(B, "B", (batch, L, N), dt, dev),
        _ptr(C, "C", (batch, L, N), dt, dev),
        _ptr(D, "D", (dim,), f32, dev, required=False),
        _ptr(z, "z", (batch, L, dim), dt, dev, required=False),
        _ptr(delta_bias, "delta_bias", (dim,), f32, dev, required=False),
        int(bool(softplus)),
        _ptr(dy, "dy", (batch, L, dim), dt, dev),
        _ptr(dfinal_state, "dfinal_state", (batch, dim, N), f32, dev, required=False),
        _ptr(out["dx"], "dx"), _ptr(out["ddelta"], "ddelta"), _ptr(out["dA"], "dA"),
        _ptr(out["dB"], "dB"), _ptr(out["dC"], "dC"), _ptr(out["dD"], "dD"),
        _ptr(out["dz"], "dz", required=False), _ptr(out["ddelta_bias"], "ddelta_bias"),
        batch, L, dim, N, code,
    ]
    lib = load_library()
    if bbar not in BBAR_MODES:
        raise ValueError(f"bbar must be one of {sorted(BBAR_MODES)}")
    if bbar != "delta":
        K = 0
        if conv_weight is not None:
            if conv_weight.dim() != 2 or conv_weight.shape[0] != dim:
                raise ValueError("conv_weight must be [dim, K]")
            K = int(conv_weight.shape[1])
            out["dconv_weight"] = torch.empty(dim, K, device=dev, dtype=f32)
            out["dconv_bias"] = (torch.empty(dim, device=dev, dtype=f32)
                                 if conv_bias is not None else None)
        if initial_state is not None:
            out["dh0"] = torch.empty(batch, dim, N, device=dev, dtype=f32)
        opts = BwdOptions(
            _ptr(initial_state, "initial_state", (batch, dim, N), f32, dev, required=False),
            _ptr(out.get("dh0"), "dh0", required=False),
            _ptr(conv_weight, "conv_weight", (dim, K), f32, dev, required=False),
            _ptr(conv_bias, "conv_bias", (dim,), f32, dev, required=False), K,
            _ptr(out.get("dconv_weight"), "dconv_weight", required=False),
            _ptr(out.get("dconv_bias"), "dconv_bias", required=False), BBAR_MODES[bbar])
        nbytes = int(lib.selscan_bwd_conv_workspace_bytes(batch, L, dim, N) if K
                     else lib.selscan_bwd_workspace_bytes(batch, L, dim, N))
        ws = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
        if stream is not None and not isinstance(stream, int):
            ws.record_stream(stream)
        eargs = args[:11] + [ctypes.byref(opts)] + args[11:] \
            + [ws.data_ptr() if nbytes else None, nbytes, _stream_ptr(stream, dev)]
        _check(lib.selscan_bwd_ex(*eargs))
        return out
    if conv_weight is not None:
        if conv_weight.dim() != 2 or conv_weight.shape[0] != dim:
            raise ValueError("conv_weight must be [dim, K]")
        K = int(conv_weight.shape[1])
        if initial_state is not None:
            out["dh0"] = torch.empty(batch, dim, N, device=dev, dtype=f32)
        out["dconv_weight"] = torch.empty(dim, K, device=dev, dtype=f32)
        out["dconv_bias"] = torch.empty(dim, device=dev, dtype=f32) if conv_bias is not None \
            else None
        nbytes = int(lib.selscan_bwd_conv_workspace_bytes(batch, L, dim, N))
        ws = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
        if stream is not None and not isinstance(stream, int):
            ws.record_stream(stream)
        cargs = ([args[0], _ptr(conv_weight, "conv_weight", (dim, K), f32, dev),
                  _ptr(conv_bias, "conv_bias", (dim,), f32, dev, required=False), K]
                 + args[1:9]
                 + [_ptr(initial_state, "initial_state", (batch, dim, N), f32, dev,
                         required=False)]
                 + args[9:19]
                 + [_ptr(out.get("dh0"), "dh0", required=False),
                    _ptr(out["dconv_weight"], "dconv_weight"),
                    _ptr(out["dconv_bias"], "dconv_bias", required=False)]
                 + args[19:]
                 + [ws.data_ptr() if nbytes else None, nbytes, _stream_ptr(stream, dev)])
        _check(lib.selscan_bwd_conv(*cargs))
        return out
    if initial_state is not None:
        out["dh0"] = torch.empty(batch, dim, N, device=dev, dtype=f32)
        nbytes = int(lib.selscan_bwd_workspace_bytes(batch, L, dim, N))
        ws = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
        if stream is not None and not isinstance(stream, int):
            ws.record_stream(stream)
        fargs = args[:9] + [_ptr(initial_state, "initial_state", (batch, dim, N), f32, dev)] \
            + args[9:19] + [_ptr(out["dh0"], "dh0")] + args[19:] \
            + [ws.data_ptr() if nbytes else None, nbytes, _stream_ptr(stream, dev)]
        _check(lib.selscan_bwd_from_state(*fargs))
        return out
    if allocate_in_library:
        _check(lib.selscan_bwd(*args, _stream_ptr(stream, dev)))
        return out
    nbytes = int(lib.selscan_bwd_workspace_bytes(batch, L, dim, N))
    ws = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
    if stream is not None and not isinstance(stream, int):
        ws.record_stream(stream)  # keep it out of the cache until that stream is done
    _check(lib.selscan_bwd_workspace(*args, ws.data_ptr() if nbytes else None, nbytes,
                                     _stream_ptr(stream, dev)))
    return out


def selscan_ssd_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus=True,
                    initial_state=None, y=None, final_state=None, return_final_state=False,
                    stream=None):
    """The scan with one scalar A per head in chunked matrix form (C ABI
    ``selscan_ssd_fwd``). x, z: [batch, L, nheads·headdim]; dt: [batch, L,
    nheads]; A, D, dt_bias: [nheads] float32; B, C: [batch, L, dstate];
    initial_state / final_state: [batch, nheads·headdim, dstate] float32.
    Returns y (or (y, final_state))."""
    torch = _torch()
    if x.dim() != 3 or dt.dim() != 3:
        raise ValueError("x must be [batch, L, dim] and dt [batch, L, nheads]")
    batch, L, dim = x.shape
    nheads = dt.shape[2]
    if nheads == 0 or dim % nheads:
        raise ValueError("dim must be a multiple of nheads")
    headdim = dim // nheads
    N = B.shape[2]
    dev, dtp = x.device, x.dtype
    code = _dtype_code(x)
    f32 = torch.float32
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty(batch, dim, N, device=dev, dtype=f32)
    lib = load_library()
    nbytes = int(lib.selscan_ssd_workspace_bytes(batch, L, nheads, headdim, N))
    ws = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
    if stream is not None and not isinstance(stream, int):
        ws.record_stream(stream)
    args = [
        _ptr(x, "x", (batch, L, dim), dtp, dev),
        _ptr(dt, "dt", (batch, L, nheads), dtp, dev),
        _ptr(A, "A", (nheads,), f32, dev),
        _ptr(B, "B", (batch, L, N), dtp, dev),
        _ptr(C, "C", (batch, L, N), dtp, dev),
        _ptr(D, "D", (nheads,), f32, dev, required=False),
        _ptr(z, "z", (batch, L, dim), dtp, dev, required=False),
        _ptr(dt_bias, "dt_bias", (nheads,), f32, dev, required=False),
        int(bool(softplus)),
        _ptr(initial_state, "initial_state", (batch, dim, N), f32, dev, required=False),
        _ptr(y, "y", (batch, L, dim), dtp, dev),
        _ptr(final_state, "final_state", (batch, dim, N), f32, dev, required=False),
        batch, L, nheads, headdim, N, code, ws.data_ptr() if nbytes else None, nbytes,
        _stream_ptr(stream, dev),
    ]
    _check(lib.selscan_ssd_fwd(*args))
    if return_final_state:
        return y, final_state
    return y


def selscan_bwd_workspace_bytes(batch: int, seqlen: int, dim: int, dstate: int) -> int:
    """Device workspace bytes ``selscan_bwd`` allocates for these sizes."""
    return int(load_library().selscan_bwd_workspace_bytes(batch, seqlen, dim, dstate))


def selscan_state_update(state, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                         softplus=True, y=None, stream=None, conv_state=None,
                         conv_weight=None, conv_bias=None, bbar="delta"):
    """One recurrent step in place on ``state`` (C ABI ``selscan_state_update``,
    or ``selscan_state_update_conv`` when ``conv_weight`` is given).

    state: [batch, dim, dstate] float32 (updated); x, delta, z: [batch, dim];
    B, C: [batch, dstate]. With the conv: x is the conv input, conv_state
    [batch, dim, 3] float32 holds the previous 3 inputs (updated), conv_weight
    [dim, K], conv_bias [dim]. Returns y [batch, dim]."""
    torch = _torch()
    if state.dim() != 3:
        raise ValueError("state must be [batch, dim, dstate]")
    batch, dim, N = state.shape
    dev, dt = x.device, x.dtype
    code = _dtype_code(x)
    if y is None:
        y = torch.empty_like(x)
    f32 = torch.float32
    tail = [
        _ptr(delta, "delta", (batch, dim), dt, dev),
        _ptr(A, "A", (dim, N), f32, dev),
        _ptr(B, "B", (batch, N), dt, dev),
        _ptr(C, "C", (batch, N), dt, dev),
        _ptr(D, "D", (dim,), f32, dev, required=False),
        _ptr(z, "z", (batch, dim), dt, dev, required=False),
        _ptr(delta_bias, "delta_bias", (dim,), f32, dev, required=False),
        int(bool(softplus)),
        _ptr(y, "y", (batch, dim), dt, dev),
        batch, dim, N, code, _stream_ptr(stream, dev),
    ]
    st = _ptr(state, "state", (batch, dim, N), f32, dev)
    if bbar != "delta":
        if bbar not in BBAR_MODES:
            raise ValueError(f"bbar must be one of {list(BBAR_MODES)}")
        has_conv = conv_weight is not None
        opts = StepOptions(
            _ptr(conv_state, "conv_state", (batch, dim, 3), f32, dev) if has_conv else None,
            _ptr(conv_weight, "conv_weight", tuple(conv_weight.shape), f32, dev)
            if has_conv else None,
            _ptr(conv_bias, "conv_bias", (dim,), f32, dev, required=False) if has_conv else None,
            int(conv_weight.shape[1]) if has_conv else 0, BBAR_MODES[bbar])
        args = [st, _ptr(x, "x", (batch, dim), dt, dev)] + tail[:8] + [ctypes.byref(opts)] \
            + tail[8:]
        _check(load_library().selscan_state_update_ex(*args))
        return y
    if conv_weight is not None:
        if conv_weight.dim() != 2 or conv_weight.shape[0] != dim:
            raise ValueError("conv_weight must be [dim, K]")
        args = [st, _ptr(conv_state, "conv_state", (batch, dim, 3), f32, dev),
                _ptr(x, "x", (batch, dim), dt, dev),
                _ptr(conv_weight, "conv_weight", tuple(conv_weight.shape), f32, dev),
                _ptr(conv_bias, "conv_bias", (dim,), f32, dev, required=False),
                int(conv_weight.shape[1])] + tail
        _check(load_library().selscan_state_update_conv(*args))
        return y
    args = [st, _ptr(x, "x", (batch, dim), dt, dev)] + tail
    _check(load_library().selscan_state_update(*args))
    return y
