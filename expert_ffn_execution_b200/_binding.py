"""ctypes binding of libstrata_moe.so: the C-ABI calls of include/strata_moe.h
under the same names.  Argument marshalling only -- every step of the layer
runs in the library's CUDA kernels.  Tensor arguments may be torch tensors
(their data_ptr() is passed) or raw integer addresses; `stream` defaults to
torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libstrata_moe.so")

OK, EINVAL, ECUDA, EUNSUPPORTED, ETIMEOUT, EBOUNDS, EOVERFLOW = range(7)
FMT_Q2_32 = 1
FMT_Q4CB_32 = 2
FMT_MXFP4_32 = 3
DTYPE_F32 = 0
DTYPE_F16 = 1
DTYPE_BF16 = 2
DECODE_MAX_T = 16
DEV_TIMEOUT = 0x1
DEV_BOUNDS = 0x2


class StrataError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} returned {status} ({status_string(status)})")
        self.status = status


class QWeights(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("num_experts", ctypes.c_int32),
                ("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("base", ctypes.c_void_p), ("expert_stride", ctypes.c_uint64)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_U64 = ctypes.c_uint64
_F = ctypes.c_float
_QW = ctypes.POINTER(QWeights)

_SIGS = {
    "strata_abi_version": (_I, []),
    "strata_status_string": (ctypes.c_char_p, [_I]),
    "strata_expert_bytes": (_U64, [_I, _I, _I]),
    "strata_read_status": (_I, [_P, _P]),
    "strata_selftest_wait": (_I, [_U64, _I, _P, _P, _P]),
    "moe_rmsnorm": (_I, [_P, _I, _I, _F, _P, _P]),
    "moe_router_topk_workspace_size": (_U64, [_I, _I, _I, _I]),
    "moe_router_topk": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _U64, _P, _P]),
    "moe_bucket_workspace_size": (_U64, [_I, _I, _I]),
    "moe_bucket": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _P, _P, _U64, _P, _P]),
    "moe_route_workspace_size": (_U64, [_I, _I, _I, _I]),
    "moe_route": (_I, [_P, _I, _I, _F, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _U64,
                       _P, _P]),
    "moe_experts_workspace_size": (_U64, [_QW, _I, _I]),
    "moe_experts": (_I, [_P, _QW, _P, _P, _P, _I, _I, _P, _P, _U64, _P, _P]),
    "moe_experts_static_scratch": (_I, [_P, _QW, _P, _P, _P, _I, _I, _P, _P, _P]),
    "moe_shared_expert_workspace_size": (_U64, [_QW, _I]),
    "moe_shared_expert": (_I, [_P, _QW, _I, _P, _P, _U64, _P, _P]),
    "moe_combine": (_I, [_P, _I, _P, _P, _P, _I, _P, _I, _I, _I, _P, _P, _P, _P]),
    "moe_gather_rows": (_I, [_P, _I, _I, _I, _P, _I, _I, _P, _I, _P, _P]),
    "moe_layer_workspace_size": (_U64, [_I, _I, _I, _QW, _QW]),
    "moe_layer_forward": (_I, [_P, _I, _P, _P, _I, _I, _QW, _QW, _F, _P, _P, _P, _P, _P, _U64,
                               _P, _P]),
}

_lib = None


def load():
    """Load the library; raise loudly if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m expert_ffn_execution_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name, rc):
    if rc != OK:
        raise StrataError(name, rc)
    return rc


def qweights(fmt: int, num_experts: int, hidden: int, inter: int, base, expert_stride: int):
    return QWeights(fmt, num_experts, hidden, inter, _ptr(base), expert_stride)


def _qw(w):
    return None if w is None else ctypes.byref(w)


# ---------------------------------------------------------------- helpers
def strata_selftest_wait(budget_cycles, mode, dev_status, dev_out, stream=None, check=True):
    rc = load().strata_selftest_wait(int(budget_cycles), int(mode), _ptr(dev_status),
                                     _ptr(dev_out), _stream(stream))
    return _check("strata_selftest_wait", rc) if check else rc


def abi_version() -> int:
    return load().strata_abi_version()


def status_string(status: int) -> str:
    return load().strata_status_string(status).decode()


def strata_expert_bytes(fmt: int, hidden: int, inter: int) -> int:
    return int(load().strata_expert_bytes(fmt, hidden, inter))


def strata_read_status(dev_status, stream=None) -> int:
    return load().strata_read_status(_ptr(dev_status), _stream(stream))


# ---------------------------------------------------------------- calls
def moe_rmsnorm(x, T, H, eps, hidden, stream=None, check=True):
    rc = load().moe_rmsnorm(_ptr(x), T, H, eps, _ptr(hidden), _stream(stream))
    return _check("moe_rmsnorm", rc) if check else rc


def moe_router_topk_workspace_size(T, H, E, k) -> int:
    return int(load().moe_router_topk_workspace_size(T, H, E, k))


def moe_router_topk(hidden, w_router, bias, T, H, E, k, topk_ids, topk_w, logits_opt,
                    workspace, ws_bytes, dev_status, stream=None, check=True):
    rc = load().moe_router_topk(_ptr(hidden), _ptr(w_router), _ptr(bias), T, H, E, k,
                                _ptr(topk_ids), _ptr(topk_w), _ptr(logits_opt), _ptr(workspace),
                                ws_bytes, _ptr(dev_status), _stream(stream))
    return _check("moe_router_topk", rc) if check else rc


def moe_bucket_workspace_size(T, k, E) -> int:
    return int(load().moe_bucket_workspace_size(T, k, E))


def moe_bucket(topk_ids, T, k, E, counts, offsets, perm, inv, active, workspace, ws_bytes,
               dev_status, stream=None, check=True):
    rc = load().moe_bucket(_ptr(topk_ids), T, k, E, _ptr(counts), _ptr(offsets), _ptr(perm),
                           _ptr(inv), _ptr(active), _ptr(workspace), ws_bytes, _ptr(dev_status),
                           _stream(stream))
    return _check("moe_bucket", rc) if check else rc


def moe_route_workspace_size(T, H, E, k) -> int:
    return int(load().moe_route_workspace_size(T, H, E, k))


def moe_route(x, T, H, eps, w_router, bias, E, k, hidden, topk_ids, topk_w, counts, offsets,
              perm, inv, active, workspace, ws_bytes, dev_status, stream=None, check=True):
    rc = load().moe_route(_ptr(x), T, H, eps, _ptr(w_router), _ptr(bias), E, k, _ptr(hidden),
                          _ptr(topk_ids), _ptr(topk_w), _ptr(counts), _ptr(offsets), _ptr(perm),
                          _ptr(inv), _ptr(active), _ptr(workspace), ws_bytes, _ptr(dev_status),
                          _stream(stream))
    return _check("moe_route", rc) if check else rc


def moe_experts_workspace_size(w: QWeights, T, k) -> int:
    return int(load().moe_experts_workspace_size(_qw(w), T, k))


def moe_experts(hidden, w: QWeights, offsets, perm, active, T, k, y, workspace, ws_bytes,
                dev_status, stream=None, check=True):
    rc = load().moe_experts(_ptr(hidden), _qw(w), _ptr(offsets), _ptr(perm), _ptr(active), T, k,
                            _ptr(y), _ptr(workspace), ws_bytes, _ptr(dev_status), _stream(stream))
    return _check("moe_experts", rc) if check else rc


def moe_experts_static_scratch(hidden, w: QWeights, offsets, perm, active, T, k, y, dev_status,
                               stream=None, check=True):
    rc = load().moe_experts_static_scratch(_ptr(hidden), _qw(w), _ptr(offsets), _ptr(perm),
                                           _ptr(active), T, k, _ptr(y), _ptr(dev_status),
                                           _stream(stream))
    return _check("moe_experts_static_scratch", rc) if check else rc


def moe_shared_expert_workspace_size(w: QWeights, T) -> int:
    return int(load().moe_shared_expert_workspace_size(_qw(w), T))


def moe_shared_expert(hidden, w: QWeights, T, y, workspace, ws_bytes, dev_status, stream=None,
                      check=True):
    rc = load().moe_shared_expert(_ptr(hidden), _qw(w), T, _ptr(y), _ptr(workspace), ws_bytes,
                                  _ptr(dev_status), _stream(stream))
    return _check("moe_shared_expert", rc) if check else rc


def moe_combine(y, y_dtype, inv, topk_w, shared_y, shared_dtype, residual, T, k, H, out,
                residual_out, dev_status, stream=None, check=True):
    rc = load().moe_combine(_ptr(y), y_dtype, _ptr(inv), _ptr(topk_w), _ptr(shared_y),
                            shared_dtype, _ptr(residual), T, k, H, _ptr(out), _ptr(residual_out),
                            _ptr(dev_status), _stream(stream))
    return _check("moe_combine", rc) if check else rc


def moe_gather_rows(src, src_dtype, n_src, H, idx, div, n, dst, dst_dtype, dev_status,
                    stream=None, check=True):
    rc = load().moe_gather_rows(_ptr(src), src_dtype, n_src, H, _ptr(idx), div, n, _ptr(dst),
                                dst_dtype, _ptr(dev_status), _stream(stream))
    return _check("moe_gather_rows", rc) if check else rc


def moe_layer_workspace_size(T, E, k, w: QWeights, shared: QWeights | None) -> int:
    return int(load().moe_layer_workspace_size(T, E, k, _qw(w), _qw(shared)))


def moe_layer_forward(x, T, w_router, bias, E, k, w: QWeights, shared: QWeights | None, eps, out,
                      residual_out, topk_ids_opt, topk_w_opt, workspace, ws_bytes, dev_status,
                      stream=None, check=True):
    rc = load().moe_layer_forward(_ptr(x), T, _ptr(w_router), _ptr(bias), E, k, _qw(w),
                                  _qw(shared), eps, _ptr(out), _ptr(residual_out),
                                  _ptr(topk_ids_opt), _ptr(topk_w_opt), _ptr(workspace),
                                  ws_bytes, _ptr(dev_status), _stream(stream))
    return _check("moe_layer_forward", rc) if check else rc
