"""Python binding of libmoeq (include/moeq.h): argument marshalling only.

Every step of the layer runs in the CUDA library; this module turns torch
tensors into device pointers, fills the C structs and checks return codes.
It raises if the library is missing: there is no fallback path.
"""
import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoeq.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_DEVICE_FAULT = 4
MOE_ERR_TIMEOUT = 5
MOE_DEV_BAD_EXPERT_ID = 0x1
MOE_DEV_BAD_SLOT = 0x2
MOE_DEV_NONFINITE = 0x4
MOE_DEV_TIMEOUT = 0x8
MOE_DT_BF16 = 0
MOE_DT_F32 = 1

# every entry point declared in include/moeq.h
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_route", "moe_expert_ffn_q4",
           "moe_expert_ffn_q2", "moe_combine_residual", "moe_layer_forward",
           "moe_get_device_status", "moe_last_error", "moe_version", "moe_layer_forward_noalloc",
           "moe_set_kernel_events", "moe_rmsnorm", "moe_layer_forward_normed",
           "moe_cache_create", "moe_cache_destroy", "moe_cache_plan", "moe_cache_stats")
NOALLOC_SCRATCH_BYTES = 4 << 20


class MoeError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"moeq status {status}: {msg}")
        self.status = status


class LayerDesc(C.Structure):
    _fields_ = [(n, C.c_int32) for n in
                ("hidden", "inter", "n_experts", "top_k", "group_size", "bits", "has_shared")]


class QMat(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scale", C.c_void_p), ("bias", C.c_void_p)]


class QExpert(C.Structure):
    _fields_ = [("gate", QMat), ("up", QMat), ("down", QMat)]


class SlotTable(C.Structure):
    _fields_ = [("slots", C.c_void_p), ("n_slots", C.c_int32)]


_lib = None


def lib():
    """Load libmoeq.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoeq.so not built at {LIB_PATH}; run "
                              "python -m quantised_expert_ffn_moe_b200.build")
        L = C.CDLL(LIB_PATH)
        vp, i32, f32p, i32p = C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p
        L.moe_workspace_size.restype = C.c_size_t
        L.moe_workspace_size.argtypes = [C.POINTER(LayerDesc), i32]
        L.moe_workspace_init.argtypes = [vp, C.c_size_t, vp]
        L.moe_route.argtypes = [C.POINTER(LayerDesc), vp, i32, vp, C.c_int, f32p, i32p, f32p, vp, vp]
        for n in ("moe_expert_ffn_q4", "moe_expert_ffn_q2"):
            getattr(L, n).argtypes = [C.POINTER(LayerDesc), vp, i32, C.POINTER(SlotTable),
                                      C.POINTER(QExpert), i32p, f32p, f32p, vp, vp]
        L.moe_combine_residual.argtypes = [C.POINTER(LayerDesc), f32p, vp, vp, vp, i32, vp, vp]
        L.moe_layer_forward.argtypes = [C.POINTER(LayerDesc), vp, vp, i32, vp, C.c_int, f32p,
                                        C.POINTER(SlotTable), C.POINTER(QExpert), vp, vp, i32p,
                                        f32p, vp, vp]
        L.moe_layer_forward_noalloc.argtypes = [C.POINTER(LayerDesc), vp, vp, i32, vp, C.c_int, f32p,
                                                C.POINTER(SlotTable), C.POINTER(QExpert), vp, vp,
                                                i32p, f32p, vp]
        L.moe_rmsnorm.argtypes = [vp, i32, i32, C.c_float, vp, vp]
        L.moe_layer_forward_normed.argtypes = [C.POINTER(LayerDesc), vp, i32, C.c_float, vp, C.c_int, f32p,
                                               C.POINTER(SlotTable), C.POINTER(QExpert), vp, vp, vp, i32p,
                                               f32p, vp, vp]
        L.moe_get_device_status.argtypes = [vp, vp, C.POINTER(C.c_int32)]
        L.moe_cache_create.argtypes = [i32, i32, C.POINTER(vp)]
        L.moe_cache_destroy.argtypes = [vp]
        L.moe_cache_destroy.restype = None
        L.moe_cache_plan.argtypes = [vp, vp, i32, vp, vp, vp, C.POINTER(C.c_int32)]
        L.moe_cache_stats.argtypes = [vp, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]
        L.moe_last_error.restype = C.c_char_p
        L.moe_version.restype = C.c_char_p
        for n in EXPORTS:
            if n not in ("moe_workspace_size", "moe_last_error", "moe_version", "moe_cache_destroy"):
                getattr(L, n).restype = C.c_int
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _check(rc):
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error().decode())


def make_desc(shape):
    """LayerDesc from a synth.LayerShape (or any object with the same fields)."""
    return LayerDesc(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.group,
                     shape.bits, int(shape.has_shared))


def qexpert(mats):
    """QExpert from {'gate': (codes, scale, bias), 'up': ..., 'down': ...} tensors."""
    def qm(k):
        c, s, b = mats[k]
        return QMat(c.data_ptr(), s.data_ptr(), b.data_ptr())
    return QExpert(qm("gate"), qm("up"), qm("down"))


class DeviceSlots:
    """HBM-resident slot table for an expert table: a device array of
    moe_qexpert (9 device pointers per expert id) plus the shared expert."""

    def __init__(self, table, n_routed):
        ptrs = []
        for e in range(n_routed):
            m = table.mats(e)
            for k in ("gate", "up", "down"):
                ptrs += [t.data_ptr() for t in m[k]]
        dev = table.gate_codes.device
        self.table = torch.tensor(ptrs, dtype=torch.int64).to(dev)
        self.struct = SlotTable(self.table.data_ptr(), n_routed)
        self.shared = qexpert(table.mats(n_routed)) if table.n > n_routed else None
        self._keep = table


def version():
    return lib().moe_version().decode()


def last_error():
    return lib().moe_last_error().decode()


def workspace_size(desc, max_tokens):
    return lib().moe_workspace_size(C.byref(desc), max_tokens)


def workspace(desc, max_tokens, device="cuda", stream=None):
    """Allocate (through torch) and zero-fill a workspace."""
    n = workspace_size(desc, max_tokens)
    if n == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "invalid layer desc")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    workspace_init(ws, stream)
    return ws


def workspace_init(ws, stream=None):
    _check(lib().moe_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def route(desc, x, w_router, ws, logit_bias=None, stream=None):
    T = x.shape[0]
    idx = torch.empty((T, desc.top_k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, desc.top_k), dtype=torch.float32, device=x.device)
    dt = MOE_DT_F32 if w_router.dtype == torch.float32 else MOE_DT_BF16
    _check(lib().moe_route(C.byref(desc), _ptr(x), T, _ptr(w_router), dt, _ptr(logit_bias),
                           _ptr(idx), _ptr(w), _ptr(ws), _stream(stream)))
    return idx, w


def expert_ffn(desc, x, slots, topk_idx, topk_w, ws, stream=None):
    """y fp32 [T][2][H]: routed weighted sum, shared expert."""
    T = x.shape[0]
    y = torch.empty((T, 2, desc.hidden), dtype=torch.float32, device=x.device)
    fn = lib().moe_expert_ffn_q4 if desc.bits == 4 else lib().moe_expert_ffn_q2
    sh = C.byref(slots.shared) if slots.shared is not None else None
    _check(fn(C.byref(desc), _ptr(x), T, C.byref(slots.struct), sh, _ptr(topk_idx), _ptr(topk_w),
              _ptr(y), _ptr(ws), _stream(stream)))
    return y


def expert_ffn_q4(desc, x, slots, topk_idx, topk_w, ws, stream=None):
    assert desc.bits == 4
    return expert_ffn(desc, x, slots, topk_idx, topk_w, ws, stream)


def expert_ffn_q2(desc, x, slots, topk_idx, topk_w, ws, stream=None):
    assert desc.bits == 2
    return expert_ffn(desc, x, slots, topk_idx, topk_w, ws, stream)


def combine_residual(desc, y, residual, x, shared_gate=None, out=None, stream=None):
    T = residual.shape[0]
    if out is None:
        out = torch.empty_like(residual)
    _check(lib().moe_combine_residual(C.byref(desc), _ptr(y), _ptr(residual), _ptr(shared_gate),
                                      _ptr(x), T, _ptr(out), _stream(stream)))
    return out


def layer_forward(desc, x, residual, w_router, slots, ws, shared_gate=None, logit_bias=None,
                  out=None, topk_idx=None, topk_w=None, stream=None):
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    dt = MOE_DT_F32 if w_router.dtype == torch.float32 else MOE_DT_BF16
    sh = C.byref(slots.shared) if slots.shared is not None else None
    _check(lib().moe_layer_forward(C.byref(desc), _ptr(x), _ptr(residual), T, _ptr(w_router), dt,
                                   _ptr(logit_bias), C.byref(slots.struct), sh, _ptr(shared_gate),
                                   _ptr(out), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                   _stream(stream)))
    return out


def layer_forward_noalloc(desc, x, residual, w_router, slots, shared_gate=None, logit_bias=None,
                          out=None, topk_idx=None, topk_w=None, stream=None):
    """moe_layer_forward_noalloc: the whole layer using the library's static
    device scratch instead of a caller-provided workspace (for callers that
    cannot allocate device memory).  The output buffer is the caller's; pass
    `out` to avoid this wrapper's own torch allocation."""
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    dt = MOE_DT_F32 if w_router.dtype == torch.float32 else MOE_DT_BF16
    sh = C.byref(slots.shared) if slots.shared is not None else None
    _check(lib().moe_layer_forward_noalloc(C.byref(desc), _ptr(x), _ptr(residual), T, _ptr(w_router),
                                           dt, _ptr(logit_bias), C.byref(slots.struct), sh,
                                           _ptr(shared_gate), _ptr(out), _ptr(topk_idx),
                                           _ptr(topk_w), _stream(stream)))
    return out


def rmsnorm(x, eps=1e-6, out=None, stream=None):
    """moe_rmsnorm: bf16 [T][H] -> bf16 [T][H] (unit weight)."""
    T, H = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(lib().moe_rmsnorm(_ptr(x), T, H, eps, _ptr(out), _stream(stream)))
    return out


def layer_forward_normed(desc, h, w_router, slots, ws, eps=1e-6, shared_gate=None, logit_bias=None,
                         out=None, xhat_out=None, topk_idx=None, topk_w=None, stream=None):
    """moe_layer_forward_normed: out = h + MoE(rmsnorm(h)); out may be h."""
    T = h.shape[0]
    if out is None:
        out = torch.empty_like(h)
    dt = MOE_DT_F32 if w_router.dtype == torch.float32 else MOE_DT_BF16
    sh = C.byref(slots.shared) if slots.shared is not None else None
    _check(lib().moe_layer_forward_normed(C.byref(desc), _ptr(h), T, eps, _ptr(w_router), dt, _ptr(logit_bias),
                                          C.byref(slots.struct), sh, _ptr(shared_gate), _ptr(out),
                                          _ptr(xhat_out), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                          _stream(stream)))
    return out


def stack_forward(layers, h, ws, eps=1e-6, logit_bias=None, xhat=None, topk=None, stream=None):
    """A chain of MoE layers, each fed the RMS-normalised running hidden state
    and adding its output to it: for each layer l, h = h + MoE_l(rmsnorm(h))
    (moe_layer_forward_normed, in place).  layers: (desc, w_router, slots,
    shared_gate) per layer; h bf16 [T][H] (updated in place and returned);
    logit_bias: None or one fp32 [T][E] tensor per layer; xhat: None or a list
    that receives each layer's normalised input; topk: None or a list that
    receives each layer's (idx, w)."""
    T = h.shape[0]
    for l, (desc, w_router, slots, sg) in enumerate(layers):
        xn = None
        if xhat is not None:
            xn = torch.empty_like(h)
            xhat.append(xn)
        idx = w = None
        if topk is not None:
            k = desc.top_k
            idx = torch.empty((T, k), dtype=torch.int32, device=h.device)
            w = torch.empty((T, k), dtype=torch.float32, device=h.device)
            topk.append((idx, w))
        layer_forward_normed(desc, h, w_router, slots, ws, eps, shared_gate=sg,
                             logit_bias=None if logit_bias is None else logit_bias[l],
                             out=h, xhat_out=xn, topk_idx=idx, topk_w=w, stream=stream)
    return h


class ExpertCache:
    """moe_cache_*: which of n_slots slots holds each expert a token routes to
    and which experts must be copied in (host policy; moves no data)."""

    def __init__(self, n_experts, n_slots):
        h = C.c_void_p()
        _check(lib().moe_cache_create(n_experts, n_slots, C.byref(h)))
        self._h = h

    def plan(self, ids):
        """ids: the token's distinct expert ids (sequence of int).  Returns
        (slot of each id, [(expert, slot) to copy in])."""
        k = len(ids)
        a = (C.c_int32 * k)(*ids)
        slot_of, fid, fsl = (C.c_int32 * k)(), (C.c_int32 * k)(), (C.c_int32 * k)()
        nf = C.c_int32()
        _check(lib().moe_cache_plan(self._h, a, k, slot_of, fid, fsl, C.byref(nf)))
        return list(slot_of), [(fid[i], fsl[i]) for i in range(nf.value)]

    def stats(self):
        h, m = C.c_int64(), C.c_int64()
        _check(lib().moe_cache_stats(self._h, C.byref(h), C.byref(m)))
        return h.value, m.value

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.moe_cache_destroy(self._h)
            self._h = None


def set_kernel_events(events):
    """moe_set_kernel_events: events = 4 torch.cuda.Event(enable_timing=True)
    (each recorded once already, so its handle exists) or None to turn off."""
    if events is None:
        _check(lib().moe_set_kernel_events(None, 0))
        return
    arr = (C.c_void_p * 4)(*[C.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_set_kernel_events(arr, 4))


def device_status(ws, stream=None):
    """(moe_status, status word); clears the word."""
    st = C.c_int32(0)
    rc = lib().moe_get_device_status(_ptr(ws), _stream(stream), C.byref(st))
    return rc, st.value
