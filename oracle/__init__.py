"""ctypes glue for the fp64 CPU oracle (plain C in moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.  It shares nothing
with the CUDA library.  All arrays are numpy, host memory.
"""
import ctypes as C
import os

import numpy as np

from . import build_oracle

_lib = None


class _QMat(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scale", C.c_void_p), ("bias", C.c_void_p)]


class _QExpert(C.Structure):
    _fields_ = [("gate", _QMat), ("up", _QMat), ("down", _QMat)]


class _Desc(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("hidden", "inter", "n_experts", "top_k", "group_size", "bits", "has_shared")]


def lib():
    """The compiled oracle.  MOE_ORACLE_LIB names another build of the same
    source (the mutation tests load deliberately broken copies this way)."""
    global _lib
    if _lib is None:
        _lib = C.CDLL(os.environ.get("MOE_ORACLE_LIB") or build_oracle.build())
        _lib.oracle_bf16_to_f64.restype = C.c_double
        _lib.oracle_bf16_to_f64.argtypes = [C.c_uint16]
        _lib.oracle_f64_to_bf16.restype = C.c_uint16
        _lib.oracle_f64_to_bf16.argtypes = [C.c_double]
        _lib.oracle_rmsnorm.restype = None
        _lib.oracle_rmsnorm.argtypes = [C.c_int32, C.c_void_p, C.c_double, C.c_void_p]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def bf16_to_f64(h):
    h = _c(h, np.uint16)
    return np.array([lib().oracle_bf16_to_f64(int(v)) for v in h.ravel()]).reshape(h.shape)


def f64_to_bf16(v):
    v = _c(v, np.float64)
    return np.array([lib().oracle_f64_to_bf16(float(x)) for x in v.ravel()],
                    dtype=np.uint16).reshape(v.shape)


def pack(bits, q):
    q = _c(q, np.uint8)
    rows, cols = q.shape
    words = np.zeros((rows, cols * bits // 32), dtype=np.uint32)
    rc = lib().oracle_pack(C.c_int(bits), _p(q), C.c_int64(rows), C.c_int64(cols), _p(words))
    if rc:
        raise ValueError(f"oracle_pack rc={rc}")
    return words


def unpack(bits, words, cols):
    words = _c(words, np.uint32)
    rows = words.shape[0]
    q = np.zeros((rows, cols), dtype=np.uint8)
    rc = lib().oracle_unpack(C.c_int(bits), _p(words), C.c_int64(rows), C.c_int64(cols), _p(q))
    if rc:
        raise ValueError(f"oracle_unpack rc={rc}")
    return q


def dequant(bits, group, codes, scale, bias, cols):
    codes, scale, bias = _c(codes, np.uint32), _c(scale, np.uint16), _c(bias, np.uint16)
    rows = codes.shape[0]
    W = np.zeros((rows, cols), dtype=np.float64)
    rc = lib().oracle_dequant(C.c_int(bits), C.c_int(group), C.c_int64(rows), C.c_int64(cols),
                              _p(codes), _p(scale), _p(bias), _p(W))
    if rc:
        raise ValueError(f"oracle_dequant rc={rc}")
    return W


def _qmv(fn, bits, group, codes, scale, bias, v):
    codes, scale, bias = _c(codes, np.uint32), _c(scale, np.uint16), _c(bias, np.uint16)
    v = _c(v, np.float64)
    rows, cols = codes.shape[0], v.shape[0]
    y = np.zeros(rows, dtype=np.float64)
    rc = fn(C.c_int(bits), C.c_int(group), C.c_int64(rows), C.c_int64(cols),
            _p(codes), _p(scale), _p(bias), _p(v), _p(y))
    if rc:
        raise ValueError(f"qmatvec rc={rc}")
    return y


def qmatvec(bits, group, codes, scale, bias, v):
    return _qmv(lib().oracle_qmatvec, bits, group, codes, scale, bias, v)


def qmatvec_grouped(bits, group, codes, scale, bias, v):
    return _qmv(lib().oracle_qmatvec_grouped, bits, group, codes, scale, bias, v)


def route(xhat, w_router, k, logit_bias=None):
    """xhat fp64 [H]; w_router fp32 or bf16-bits(uint16) [E][H]."""
    xhat = _c(xhat, np.float64)
    is_f32 = w_router.dtype == np.float32
    w_router = _c(w_router, np.float32 if is_f32 else np.uint16)
    E, H = w_router.shape
    logits = np.zeros(E)
    idx = np.zeros(k, dtype=np.int32)
    w = np.zeros(k)
    lb = None if logit_bias is None else _c(logit_bias, np.float64)
    rc = lib().oracle_route(C.c_int32(E), C.c_int32(H), C.c_int32(k), _p(xhat), _p(w_router),
                            C.c_int(1 if is_f32 else 0), _p(lb), _p(logits), _p(idx), _p(w))
    if rc:
        raise ValueError(f"oracle_route rc={rc}")
    return logits, idx, w


class Expert:
    """Host copy of one quantised expert: dict of numpy arrays
    gate/up/down -> (codes uint32 [rows][words], scale uint16, bias uint16)."""

    def __init__(self, gate, up, down):
        self.mats = {"gate": tuple(_c(a, t) for a, t in zip(gate, (np.uint32, np.uint16, np.uint16))),
                     "up": tuple(_c(a, t) for a, t in zip(up, (np.uint32, np.uint16, np.uint16))),
                     "down": tuple(_c(a, t) for a, t in zip(down, (np.uint32, np.uint16, np.uint16)))}

    def cstruct(self):
        def qm(m):
            c, s, b = self.mats[m]
            return _QMat(c.ctypes.data, s.ctypes.data, b.ctypes.data)
        return _QExpert(qm("gate"), qm("up"), qm("down"))


def expert_ffn(bits, group, H, I, expert, xhat):
    xhat = _c(xhat, np.float64)
    h = np.zeros(I)
    y = np.zeros(H)
    st = expert.cstruct()
    rc = lib().oracle_expert_ffn(C.c_int(bits), C.c_int(group), C.c_int32(H), C.c_int32(I),
                                 C.byref(st), _p(xhat), _p(h), _p(y))
    if rc:
        raise ValueError(f"oracle_expert_ffn rc={rc}")
    return h, y


def layer_forward(desc, xhat, residual, w_router, experts, shared=None, shared_gate=None,
                  logit_bias=None):
    """desc: dict(hidden, inter, n_experts, top_k, group_size, bits, has_shared).
    xhat, residual: bf16 bits uint16 [T][H].  experts: dict expert id -> Expert
    (only the ones that will be selected need be present).  Returns
    (out fp64 [T][H], idx int32 [T][k], w fp64 [T][k], gamma fp64 [T])."""
    d = _Desc(*(int(desc[n]) for n in
                ("hidden", "inter", "n_experts", "top_k", "group_size", "bits", "has_shared")))
    xhat = _c(xhat, np.uint16)
    residual = _c(residual, np.uint16)
    T, H = xhat.shape
    E, k = d.n_experts, d.top_k
    is_f32 = w_router.dtype == np.float32
    w_router = _c(w_router, np.float32 if is_f32 else np.uint16)
    table = (_QExpert * E)()
    keep = []
    for e, ex in experts.items():
        table[e] = ex.cstruct()
        keep.append(ex)
    sh = shared.cstruct() if shared is not None else None
    sg = None if shared_gate is None else _c(shared_gate, np.uint16)
    lb = None if logit_bias is None else _c(logit_bias, np.float64)
    out = np.zeros((T, H))
    idx = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k))
    gamma = np.zeros(T)
    rc = lib().oracle_layer_forward(C.byref(d), C.c_int32(T), _p(xhat), _p(residual), _p(w_router),
                                    C.c_int(1 if is_f32 else 0), _p(lb), table,
                                    C.byref(sh) if sh is not None else None, _p(sg),
                                    _p(out), _p(idx), _p(w), _p(gamma))
    if rc:
        raise ValueError(f"oracle_layer_forward rc={rc}")
    return out, idx, w, gamma


def rmsnorm(x, eps=1e-6):
    x = _c(x, np.float64)
    out = np.zeros_like(x)
    lib().oracle_rmsnorm(C.c_int32(x.shape[0]), _p(x), C.c_double(eps), _p(out))
    return out
