"""ctypes wrapper of the plain C oracle (strata_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the package's smoke check
and by bench.py's CPU-baseline / reference leg, never by the product path.
It shares no code with the CUDA library.  Every function takes and returns
numpy arrays; bf16/fp16 values travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "strata_oracle.c")
_LIB = os.path.join(_HERE, "libstrata_oracle.so")
# A test may point the wrapper at a separately compiled copy of the oracle
# (the mutation test plants mistakes in such a copy to show the pins fail).
_LIB_OVERRIDE = os.environ.get("STRATA_ORACLE_LIB")

FMT_Q2 = 1
FMT_Q4CB = 2
FMT_MXFP4 = 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP over tokens, no FMA
    contraction so the fp32 accumulation order is the written one)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-Wall",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            L = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        L.oracle_version.restype = ctypes.c_int
        L.oracle_expert_bytes.restype = ctypes.c_size_t
        L.oracle_expert_bytes.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oracle_dequant_row.restype = ctypes.c_int
        L.oracle_dequant_row.argtypes = [ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, P]
        L.oracle_rmsnorm.restype = None
        L.oracle_rmsnorm.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_double, P]
        L.oracle_router_logits.restype = None
        L.oracle_router_logits.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        L.oracle_topk.restype = ctypes.c_int
        L.oracle_topk.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_bucket.restype = ctypes.c_int
        L.oracle_bucket.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
        L.oracle_expert_ffn.restype = ctypes.c_int
        L.oracle_expert_ffn.argtypes = [ctypes.c_int, P, ctypes.c_int, ctypes.c_int, P, P,
                                        ctypes.c_int]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     P, P, P]
        L.oracle_moe_layer.restype = ctypes.c_int
        L.oracle_moe_layer.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, P,
                                       ctypes.c_int, P, P, P, P, P, P, P, P, P, ctypes.c_int]
        L.oracle_num_threads.restype = ctypes.c_int
        del i32
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


def expert_bytes(fmt: int, H: int, I: int) -> int:
    return int(lib().oracle_expert_bytes(fmt, H, I))


def dequant_row(fmt: int, blob, H: int, I: int, which: int, row: int) -> np.ndarray:
    blob = _c(blob, np.uint8)
    K = H if which < 2 else I
    out = np.empty(K, np.float32)
    rc = lib().oracle_dequant_row(fmt, _p(blob), H, I, which, row, _p(out))
    if rc:
        raise ValueError("oracle_dequant_row: bad argument")
    return out


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    x = _c(x, np.float32)
    T, H = x.shape
    out = np.empty((T, H), np.uint16)
    lib().oracle_rmsnorm(_p(x), T, H, float(eps), _p(out))
    return out


def router_logits(hidden, wr, bias=None) -> np.ndarray:
    hidden = _c(hidden, np.uint16)
    wr = _c(wr, np.uint16)
    T, H = hidden.shape
    E = wr.shape[1]
    bias = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float32)
    lib().oracle_router_logits(_p(hidden), _p(wr), _p(bias), T, H, E, _p(out))
    return out


def topk(logits, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    if lib().oracle_topk(_p(logits), T, E, k, _p(ids), _p(w)):
        raise ValueError("oracle_topk: bad argument")
    return ids, w


def bucket(ids, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    P = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(P, np.int32)
    inv = np.empty(P, np.int32)
    if lib().oracle_bucket(_p(ids), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv)):
        raise ValueError("oracle_bucket: bad argument")
    return counts, offsets, perm, inv


def expert_ffn(fmt: int, blob, H: int, I: int, x_row, acc64: bool = False) -> np.ndarray:
    blob = _c(blob, np.uint8)
    x_row = _c(x_row, np.uint16)
    y = np.empty(H, np.float32)
    if lib().oracle_expert_ffn(fmt, _p(blob), H, I, _p(x_row), _p(y), int(acc64)):
        raise ValueError("oracle_expert_ffn: bad argument")
    return y


def combine(y_pairs, w, shared=None, residual=None):
    y_pairs = _c(y_pairs, np.float32)
    w = _c(w, np.float32)
    T, k = w.shape
    H = y_pairs.shape[1]
    shared = None if shared is None else _c(shared, np.float32)
    residual = None if residual is None else _c(residual, np.float32)
    out_f32 = np.empty((T, H), np.float32)
    out_bf16 = np.empty((T, H), np.uint16)
    res_out = None if residual is None else np.empty((T, H), np.float32)
    lib().oracle_combine(_p(y_pairs), _p(w), _p(shared), _p(residual), T, k, H,
                         _p(out_f32), _p(out_bf16), _p(res_out))
    return out_f32, out_bf16, res_out


def moe_layer(hidden, wr, bias, E: int, k: int, fmt: int, I: int, blobs,
              shared_fmt: int = 0, shared_blob=None, forced_ids=None, residual=None,
              acc64: bool = False) -> dict:
    """The whole layer on T tokens.  `blobs` is a 2-D uint8 array [E, bytes]
    or a dict {expert id: 1-D uint8 array} holding at least the routed
    experts."""
    hidden = _c(hidden, np.uint16)
    wr = _c(wr, np.uint16)
    T, H = hidden.shape
    bias = None if bias is None else _c(bias, np.float32)
    keep = []
    ptrs = (ctypes.c_void_p * E)()
    if isinstance(blobs, dict):
        for e, b in blobs.items():
            b = _c(b, np.uint8)
            keep.append(b)
            ptrs[int(e)] = b.ctypes.data
    else:
        blobs = _c(blobs, np.uint8)
        keep.append(blobs)
        stride = blobs.shape[1]
        for e in range(E):
            ptrs[e] = blobs.ctypes.data + e * stride
    sb = None if shared_blob is None else _c(shared_blob, np.uint8).reshape(-1)
    fi = None if forced_ids is None else _c(forced_ids, np.int32)
    residual = None if residual is None else _c(residual, np.float32)
    logits = np.empty((T, E), np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    out_f32 = np.empty((T, H), np.float32)
    out_bf16 = np.empty((T, H), np.uint16)
    res_out = None if residual is None else np.empty((T, H), np.float32)
    rc = lib().oracle_moe_layer(_p(hidden), T, H, _p(wr), _p(bias), E, k, fmt, I,
                                ctypes.cast(ptrs, ctypes.c_void_p), int(shared_fmt), _p(sb),
                                _p(fi), _p(residual), _p(logits), _p(ids), _p(w),
                                _p(out_f32), _p(out_bf16), _p(res_out), int(acc64))
    if rc:
        raise ValueError("oracle_moe_layer: bad argument or missing expert blob")
    return dict(logits=logits, ids=ids, w=w, out_f32=out_f32, out_bf16=out_bf16,
                residual_out=res_out)


# ------------------------------------------------------------ bit helpers
def bf16_bits_to_f32(u16) -> np.ndarray:
    u = np.asarray(u16, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32)


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bits (numpy, for building inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)
