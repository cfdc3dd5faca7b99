"""Python binding of the C ABI in include/flashipa_b200.h.

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch provides device memory and streams.  The library must be
built (`python -m rna_structure_models_b200.build`); if it is missing, the
first call raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflashipa_b200.so")

IPA_DTYPE_F32, IPA_DTYPE_F64, IPA_DTYPE_BOOL, IPA_DTYPE_F16, IPA_DTYPE_I32 = 0, 1, 2, 3, 4
STATUS = {0: "IPA_OK", 1: "IPA_ERR_NULL", 2: "IPA_ERR_SHAPE", 3: "IPA_ERR_STRIDE_ALIGN",
          4: "IPA_ERR_DTYPE", 5: "IPA_ERR_WORKSPACE", 6: "IPA_ERR_UNSUPPORTED", 7: "IPA_ERR_CUDA",
          8: "IPA_ERR_TIMEOUT"}
EXPORTED = ("ipa_attn_workspace_size", "ipa_attn_fwd", "ipa_attn_prologue", "ipa_attn_core",
            "ipa_attn_fwd_train", "ipa_attn_bwd_workspace_size", "ipa_attn_bwd",
            "ipa_attn_host_staging_size", "ipa_attn_fwd_host", "ipa_attn_host_packed_layout",
            "ipa_attn_fwd_host_packed",
            "geo_attn_workspace_size", "geo_attn_fwd", "geo_attn_fwd_static",
            "geo_attn_bwd_workspace_size", "geo_attn_bwd",
            "meet_attn_workspace_size", "meet_attn_fwd", "ipa_frames_from_backbone", "ipa_linear_workspace_size",
            "ipa_linear_fwd", "ipa_module_workspace_size", "ipa_module_fwd", "ipa_status_string",
            "ipa_device_error_status", "ipa_version", "ipa_knn_distogram")


class IpaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("size", ctypes.c_int64 * 6), ("stride", ctypes.c_int64 * 6)]


class IpaParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32),
                ("C", ctypes.c_int32), ("Pq", ctypes.c_int32), ("Pv", ctypes.c_int32),
                ("R", ctypes.c_int32), ("Cz", ctypes.c_int32), ("w_L", ctypes.c_float),
                ("w_C", ctypes.c_float), ("scalar_scale", ctypes.c_float)]


class GeoParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("H", ctypes.c_int32),
                ("M", ctypes.c_int32), ("Cout", ctypes.c_int32)]


GEO_GRADS = ("q_direction", "k_direction", "q_point", "k_point", "values", "direction_scale",
             "distance_scale", "output_weight", "output_bias", "rotation", "translation")


class GeoGrads(ctypes.Structure):
    _fields_ = [(n, IpaTensor) for n in GEO_GRADS]


IPA_GRADS = ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "w_bias", "gamma")


class IpaGrads(ctypes.Structure):
    _fields_ = [(n, IpaTensor) for n in IPA_GRADS]


class MeetParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32),
                ("C", ctypes.c_int32)]


class ModuleParams(ctypes.Structure):
    _fields_ = [("core", IpaParams), ("c_s", ctypes.c_int32)]


class IpaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{STATUS.get(code, code)}{': ' + what if what else ''}")


_lib = None


def library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m rna_structure_models_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    T = P(IpaTensor)
    lib.ipa_attn_workspace_size.argtypes = [P(IpaParams)]
    lib.ipa_attn_workspace_size.restype = ctypes.c_size_t
    lib.ipa_attn_fwd.argtypes = [P(IpaParams)] + [T] * 14 + [ctypes.c_void_p, ctypes.c_size_t,
                                                            ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_attn_fwd.restype = ctypes.c_int
    lib.ipa_attn_prologue.argtypes = [P(IpaParams)] + [T] * 13 + [ctypes.c_void_p, ctypes.c_size_t,
                                                                 ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_attn_prologue.restype = ctypes.c_int
    lib.ipa_attn_core.argtypes = [P(IpaParams), T, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                  ctypes.c_void_p]
    lib.ipa_attn_core.restype = ctypes.c_int
    lib.ipa_attn_fwd_train.argtypes = [P(IpaParams)] + [T] * 16 + [ctypes.c_void_p, ctypes.c_size_t,
                                                                  ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_attn_fwd_train.restype = ctypes.c_int
    lib.ipa_attn_host_staging_size.argtypes = [P(IpaParams)]
    lib.ipa_attn_host_staging_size.restype = ctypes.c_size_t
    lib.ipa_attn_fwd_host.argtypes = [P(IpaParams)] + [T] * 14 + [ctypes.c_void_p, ctypes.c_size_t,
                                                                 ctypes.c_void_p, ctypes.c_size_t,
                                                                 ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_attn_fwd_host.restype = ctypes.c_int
    lib.ipa_attn_host_packed_layout.argtypes = [P(IpaParams), P(ctypes.c_size_t * 13)]
    lib.ipa_attn_host_packed_layout.restype = ctypes.c_size_t
    lib.ipa_attn_fwd_host_packed.argtypes = [P(IpaParams), ctypes.c_void_p, ctypes.c_size_t, T, ctypes.c_void_p,
                                             ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                             ctypes.c_void_p]
    lib.ipa_attn_fwd_host_packed.restype = ctypes.c_int
    lib.ipa_attn_bwd_workspace_size.argtypes = [P(IpaParams)]
    lib.ipa_attn_bwd_workspace_size.restype = ctypes.c_size_t
    lib.ipa_attn_bwd.argtypes = [P(IpaParams)] + [T] * 17 + [P(IpaGrads), ctypes.c_void_p, ctypes.c_size_t,
                                                            ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_attn_bwd.restype = ctypes.c_int
    lib.geo_attn_workspace_size.argtypes = [P(GeoParams)]
    lib.geo_attn_workspace_size.restype = ctypes.c_size_t
    lib.geo_attn_fwd.argtypes = [P(GeoParams)] + [T] * 16 + [ctypes.c_void_p, ctypes.c_size_t,
                                                            ctypes.c_void_p, ctypes.c_void_p]
    lib.geo_attn_fwd.restype = ctypes.c_int
    lib.meet_attn_workspace_size.argtypes = [P(MeetParams)]
    lib.meet_attn_workspace_size.restype = ctypes.c_size_t
    lib.meet_attn_fwd.argtypes = [P(MeetParams)] + [T] * 8 + [ctypes.c_void_p, ctypes.c_size_t,
                                                              ctypes.c_void_p, ctypes.c_void_p]
    lib.meet_attn_fwd.restype = ctypes.c_int
    lib.ipa_frames_from_backbone.argtypes = [ctypes.c_int32, ctypes.c_int32] + [T] * 5 + [ctypes.c_void_p]
    lib.ipa_frames_from_backbone.restype = ctypes.c_int
    lib.geo_attn_bwd_workspace_size.argtypes = [P(GeoParams)]
    lib.geo_attn_bwd_workspace_size.restype = ctypes.c_size_t
    lib.geo_attn_bwd.argtypes = [P(GeoParams)] + [T] * 16 + [P(GeoGrads), ctypes.c_void_p, ctypes.c_size_t,
                                                             ctypes.c_void_p, ctypes.c_void_p]
    lib.geo_attn_bwd.restype = ctypes.c_int
    lib.ipa_linear_workspace_size.argtypes = [ctypes.c_int32] * 3
    lib.ipa_linear_workspace_size.restype = ctypes.c_size_t
    lib.ipa_linear_fwd.argtypes = [ctypes.c_int32] * 3 + [T] * 4 + [ctypes.c_void_p, ctypes.c_size_t,
                                                                  ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_linear_fwd.restype = ctypes.c_int
    lib.ipa_module_workspace_size.argtypes = [P(ModuleParams)]
    lib.ipa_module_workspace_size.restype = ctypes.c_size_t
    lib.ipa_module_fwd.argtypes = [P(ModuleParams)] + [T] * 14 + [ctypes.c_void_p, ctypes.c_size_t,
                                                                  ctypes.c_void_p, ctypes.c_void_p]
    lib.ipa_module_fwd.restype = ctypes.c_int
    lib.ipa_knn_distogram.argtypes = [ctypes.c_int32] * 4 + [T, T, ctypes.POINTER(ctypes.c_float), T, T, T,
                                                             ctypes.c_void_p]
    lib.ipa_knn_distogram.restype = ctypes.c_int
    lib.ipa_status_string.argtypes = [ctypes.c_int]
    lib.ipa_status_string.restype = ctypes.c_char_p
    lib.ipa_device_error_status.argtypes = [ctypes.c_int32]
    lib.ipa_device_error_status.restype = ctypes.c_int
    lib.ipa_version.argtypes = []
    lib.ipa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


_DT = {torch.float32: IPA_DTYPE_F32, torch.float64: IPA_DTYPE_F64, torch.bool: IPA_DTYPE_BOOL,
       torch.uint8: IPA_DTYPE_BOOL, torch.float16: IPA_DTYPE_F16, torch.int32: IPA_DTYPE_I32}


def tensor_desc(t: Optional[torch.Tensor]) -> IpaTensor:
    """Describe a torch tensor (no copy; strides in elements)."""
    d = IpaTensor()
    if t is None:
        d.data = None
        return d
    if t.dim() > 6:
        raise ValueError("at most 6 dimensions")
    d.data = t.data_ptr() if t.numel() > 0 else None
    d.dtype = _DT.get(t.dtype, -1)
    d.ndim = t.dim()
    for i, (s, st) in enumerate(zip(t.shape, t.stride())):
        d.size[i] = s
        d.stride[i] = st
    return d


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors (use ipa_attn_host for host buffers)")


def ipa_defaults(C: int, Pq: int) -> dict:
    """AlphaFold-2 IPA logit weights."""
    return {"w_L": math.sqrt(1.0 / 3.0), "w_C": math.sqrt(2.0 / (9.0 * Pq)),
            "scalar_scale": 1.0 / math.sqrt(C)}


def ipa_params(B, L, H, C, Pq, Pv, R, Cz, w_L=None, w_C=None, scalar_scale=None) -> IpaParams:
    d = ipa_defaults(C, Pq)
    return IpaParams(B, L, H, C, Pq, Pv, R, Cz,
                     d["w_L"] if w_L is None else w_L,
                     d["w_C"] if w_C is None else w_C,
                     d["scalar_scale"] if scalar_scale is None else scalar_scale)


def ipa_workspace_bytes(p: IpaParams) -> int:
    return int(library().ipa_attn_workspace_size(ctypes.byref(p)))


class IpaPlan:
    """Reusable launch state for one problem shape: params, workspace and a
    device error word allocated once (by torch), so repeated calls allocate
    nothing."""

    def __init__(self, B, L, H, C=16, Pq=4, Pv=8, R=2, Cz=128, device="cuda", **consts):
        self.params = ipa_params(B, L, H, C, Pq, Pv, R, Cz, **consts)
        nbytes = ipa_workspace_bytes(self.params)
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)
        self.F = C + 4 * Pv + Cz

    def __call__(self, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask,
                 out=None, stream=None):
        p = self.params
        _require_cuda(q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask)
        if out is None:
            out = torch.empty((p.B, p.L, p.H, self.F), dtype=torch.float32, device=q.device)
        descs = [tensor_desc(t) for t in (q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2,
                                          w_bias, gamma, mask, out)]
        st = library().ipa_attn_fwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                    ctypes.c_void_p(self.workspace.data_ptr()),
                                    ctypes.c_size_t(self.workspace.numel()),
                                    ctypes.c_void_p(_stream_ptr(stream)),
                                    ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def prologue(self, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask,
                 stream=None):
        """Stage 1 only: frames applied, augmented operands written to the workspace."""
        p = self.params
        _require_cuda(q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask)
        descs = [tensor_desc(t) for t in (q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2,
                                          w_bias, gamma, mask)]
        st = library().ipa_attn_prologue(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                         ctypes.c_void_p(self.workspace.data_ptr()),
                                         ctypes.c_size_t(self.workspace.numel()),
                                         ctypes.c_void_p(_stream_ptr(stream)),
                                         ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())

    def core(self, out, stream=None):
        """Stage 2 only: the fused attention pass from the workspace into `out`."""
        d = tensor_desc(out)
        st = library().ipa_attn_core(ctypes.byref(self.params), ctypes.byref(d),
                                     ctypes.c_void_p(self.workspace.data_ptr()),
                                     ctypes.c_size_t(self.workspace.numel()),
                                     ctypes.c_void_p(_stream_ptr(stream)),
                                     ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def train(self, q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask,
              out=None, lse=None, u_agg=None, stream=None):
        """Training forward: the output plus the log-sum-exp of the logits
        [B, H, L] and the pair aggregate U [B, L, H, R, Cz] that the gradient
        pass needs.  Returns (out, lse, u_agg)."""
        p = self.params
        _require_cuda(q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2, w_bias, gamma, mask)
        dev = q.device
        if out is None:
            out = torch.empty((p.B, p.L, p.H, self.F), dtype=torch.float32, device=dev)
        if lse is None:
            lse = torch.empty((p.B, p.H, p.L), dtype=torch.float32, device=dev)
        if u_agg is None:
            u_agg = torch.empty((p.B, p.L, p.H, p.R, p.Cz), dtype=torch.float32, device=dev)
        descs = [tensor_desc(t) for t in (q, k, v, q_pts, k_pts, v_pts, rot, trans, z1, z2,
                                          w_bias, gamma, mask, out, lse, u_agg)]
        st = library().ipa_attn_fwd_train(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                          ctypes.c_void_p(self.workspace.data_ptr()),
                                          ctypes.c_size_t(self.workspace.numel()),
                                          ctypes.c_void_p(_stream_ptr(stream)),
                                          ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out, lse, u_agg

    def check(self):
        """Synchronise and raise if a kernel reported a device-side error."""
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


class IpaGradPlan:
    """Gradients of the fused IPA core for one problem shape; the plan owns
    the workspace (linear in L) and a device error word."""

    def __init__(self, B, L, H, C=16, Pq=4, Pv=8, R=2, Cz=128, device="cuda", **consts):
        self.params = ipa_params(B, L, H, C, Pq, Pv, R, Cz, **consts)
        nbytes = int(library().ipa_attn_bwd_workspace_size(ctypes.byref(self.params)))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, inp: dict, out, lse, u_agg, g_out, *, grads: Optional[dict] = None, stream=None) -> dict:
        """inp: the forward inputs (IPA_INPUTS); out, lse, u_agg: the training
        forward's results; g_out: upstream gradient of out.  Returns the
        gradients of sum(g_out * out) keyed like IPA_GRADS."""
        p = self.params
        _require_cuda(*[inp[n] for n in IPA_INPUTS], out, lse, u_agg, g_out)
        if grads is None:
            grads = {n: torch.empty(tuple(inp[n].shape), dtype=torch.float32, device=out.device) for n in IPA_GRADS}
        descs = [tensor_desc(inp[n]) for n in IPA_INPUTS] + [tensor_desc(t) for t in (out, lse, u_agg, g_out)]
        gs = IpaGrads(*[tensor_desc(grads[n]) for n in IPA_GRADS])
        st = library().ipa_attn_bwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs], ctypes.byref(gs),
                                    ctypes.c_void_p(self.workspace.data_ptr()),
                                    ctypes.c_size_t(self.workspace.numel()),
                                    ctypes.c_void_p(_stream_ptr(stream)),
                                    ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return grads

    def check(self):
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


IPA_INPUTS = ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "w_bias",
              "gamma", "mask")


def ipa_attn(inp: dict, *, out=None, stream=None, check: bool = True, **consts):
    """Fused IPA core on CUDA tensors given in a dict keyed like IPA_INPUTS."""
    q = inp["q"]
    B, L, H, C = q.shape
    Pq, Pv = inp["q_pts"].shape[3], inp["v_pts"].shape[3]
    R, Cz = inp["z1"].shape[2], inp["z1"].shape[3]
    plan = IpaPlan(B, L, H, C, Pq, Pv, R, Cz, device=q.device, **consts)
    res = plan(*[inp[n] for n in IPA_INPUTS], out=out, stream=stream)
    if check:
        plan.check()
    return res


def _dims_of(inp: dict):
    q = inp["q"]
    B, L, H, C = q.shape
    return B, L, H, C, inp["q_pts"].shape[3], inp["v_pts"].shape[3], inp["z1"].shape[2], inp["z1"].shape[3]


def ipa_attn_train(inp: dict, *, stream=None, check: bool = True, **consts):
    """Training forward on CUDA tensors: (out, lse, u_agg)."""
    plan = IpaPlan(*_dims_of(inp), device=inp["q"].device, **consts)
    res = plan.train(*[inp[n] for n in IPA_INPUTS], stream=stream)
    if check:
        plan.check()
    return res


def ipa_attn_backward(inp: dict, out, lse, u_agg, g_out, *, stream=None, check: bool = True, **consts) -> dict:
    """Gradients of sum(g_out * out) with respect to every float input."""
    plan = IpaGradPlan(*_dims_of(inp), device=inp["q"].device, **consts)
    res = plan(inp, out, lse, u_agg, g_out, stream=stream)
    if check:
        plan.check()
    return res


def ipa_attn_host(inp: dict, plan: Optional[IpaPlan] = None, device="cuda", stream=None, out=None):
    """End-to-end call on HOST tensors: copies the inputs to the device (from
    pinned memory when they are pinned), runs the fused core, copies the
    result back into a pinned host tensor (`out` if given, else one cached on
    the plan).  Device staging buffers are cached on the plan and reused by
    later calls with the same shapes.  Returns (out_host, plan); the copy
    back is asynchronous on the current stream."""
    q = inp["q"]
    B, L, H, C = q.shape
    if plan is None:
        plan = IpaPlan(B, L, H, C, inp["q_pts"].shape[3], inp["v_pts"].shape[3],
                       inp["z1"].shape[2], inp["z1"].shape[3], device=device)
    cache = plan.__dict__.setdefault("_host_cache", {})
    dev = {}
    for n in IPA_INPUTS:
        t = inp[n]
        key = (n, tuple(t.shape), t.stride(), t.dtype)
        buf = cache.get(key)
        if buf is None:
            buf = cache[key] = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=device)
        buf.copy_(t, non_blocking=True)
        dev[n] = buf
    okey = ("out", B, L, H, plan.F)
    if okey not in cache:
        cache[okey] = torch.empty((B, L, H, plan.F), dtype=torch.float32, device=device)
    res = plan(*[dev[n] for n in IPA_INPUTS], out=cache[okey], stream=stream)
    if out is None:
        hkey = ("host", B, L, H, plan.F)
        if hkey not in cache:
            cache[hkey] = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
        out = cache[hkey]
    out.copy_(res, non_blocking=True)
    return out, plan


class IpaHostCalls:
    """Calls of the C entry point ipa_attn_fwd_host (host buffers in, host
    result out; the copies and kernels are enqueued by the library) on
    `slots` streams, each with its own device staging, workspace and error
    word, so that one call's copies overlap another call's kernels."""

    def __init__(self, B, L, H, C=16, Pq=4, Pv=8, R=2, Cz=128, slots=2, device="cuda", **consts):
        self.params = ipa_params(B, L, H, C, Pq, Pv, R, Cz, **consts)
        lib = library()
        ns = int(lib.ipa_attn_host_staging_size(ctypes.byref(self.params)))
        nw = int(lib.ipa_attn_workspace_size(ctypes.byref(self.params)))
        if ns == 0 or nw == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.device = torch.device(device)
        self.staging = [torch.empty(ns, dtype=torch.uint8, device=device) for _ in range(slots)]
        self.workspace = [torch.empty(nw, dtype=torch.uint8, device=device) for _ in range(slots)]
        self.dev_err = torch.zeros(slots, dtype=torch.int32, device=device)
        self.streams = [torch.cuda.Stream(self.device) for _ in range(slots)]
        self.F = C + 4 * Pv + Cz

    def call(self, inp: dict, out, slot: int = 0):
        """Enqueue one call on slot `slot`'s stream (host tensors, contiguous)."""
        descs = [tensor_desc(inp[n]) for n in IPA_INPUTS] + [tensor_desc(out)]
        st = library().ipa_attn_fwd_host(ctypes.byref(self.params), *[ctypes.byref(d) for d in descs],
                                         ctypes.c_void_p(self.staging[slot].data_ptr()),
                                         ctypes.c_size_t(self.staging[slot].numel()),
                                         ctypes.c_void_p(self.workspace[slot].data_ptr()),
                                         ctypes.c_size_t(self.workspace[slot].numel()),
                                         ctypes.c_void_p(self.streams[slot].cuda_stream),
                                         ctypes.c_void_p(self.dev_err[slot:].data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())

    def packed_layout(self):
        """(size in bytes, byte offsets of the 13 inputs) of the packed host
        buffer ipa_attn_fwd_host_packed reads."""
        offs = (ctypes.c_size_t * 13)()
        n = int(library().ipa_attn_host_packed_layout(ctypes.byref(self.params), ctypes.byref(offs)))
        if n == 0:
            raise IpaError(2, "shape mismatch")
        return n, [int(o) for o in offs]

    def pack(self, inp: dict, buf=None):
        """Copies the 13 host inputs (contiguous; fp32, mask bool / uint8) into
        one page-locked byte buffer at the packed offsets (a host-side copy,
        done once per set of inputs, outside any timed call)."""
        n, offs = self.packed_layout()
        if buf is None:
            buf = torch.zeros(n, dtype=torch.uint8, pin_memory=True)
        for name, off in zip(IPA_INPUTS, offs):
            t = inp[name].contiguous()
            if t.dtype == torch.bool:
                t = t.to(torch.uint8)
            b = t.reshape(-1).view(torch.uint8)
            buf[off:off + b.numel()].copy_(b)
        return buf

    def call_packed(self, buf, out, slot: int = 0):
        """Enqueue one ipa_attn_fwd_host_packed call on slot `slot`'s stream."""
        od = tensor_desc(out)
        st = library().ipa_attn_fwd_host_packed(ctypes.byref(self.params), ctypes.c_void_p(buf.data_ptr()),
                                                ctypes.c_size_t(buf.numel()), ctypes.byref(od),
                                                ctypes.c_void_p(self.staging[slot].data_ptr()),
                                                ctypes.c_size_t(self.staging[slot].numel()),
                                                ctypes.c_void_p(self.workspace[slot].data_ptr()),
                                                ctypes.c_size_t(self.workspace[slot].numel()),
                                                ctypes.c_void_p(self.streams[slot].cuda_stream),
                                                ctypes.c_void_p(self.dev_err[slot:].data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())

    def run(self, inputs, outputs):
        """Calls k = 0, 1, ... on slot k mod slots; waits for all of them."""
        for k, (inp, out) in enumerate(zip(inputs, outputs)):
            self.call(inp, out, k % len(self.streams))
        for s in self.streams:
            s.synchronize()
        return outputs

    def check(self):
        v = self.dev_err.cpu()
        if int(v.abs().sum()) != 0:
            self.dev_err.zero_()
            code = int(v[v != 0][0])
            raise IpaError(int(library().ipa_device_error_status(code)), f"device error code {code}")


class IpaHostPipeline:
    """Many calls on HOST buffers with the transfers overlapped across calls:
    call k's inputs go up on a copy stream while call k-1 computes and call
    k-2's result comes down on a second copy stream (PCIe carries both
    directions at once).  Two device staging sets; events order every reuse.
    Each call's copies and kernels are the same as ipa_attn_host's."""

    def __init__(self, plan: IpaPlan, device="cuda"):
        self.plan = plan
        self.device = torch.device(device)
        self.up, self.comp, self.down = (torch.cuda.Stream(self.device) for _ in range(3))
        self.sets = [{}, {}]
        self.outs = [None, None]
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]  # noqa: E731
        self.uploaded, self.consumed, self.computed, self.downloaded = ev(), ev(), ev(), ev()

    def _stage(self, s, inp):
        d = self.sets[s]
        for n in IPA_INPUTS:
            t = inp[n]
            buf = d.get(n)
            if buf is None or buf.shape != t.shape or buf.stride() != t.stride() or buf.dtype != t.dtype:
                buf = d[n] = torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=self.device)
            buf.copy_(t, non_blocking=True)
        return d

    def run(self, inputs, outputs, stream=None):
        """inputs: list of dicts of pinned host tensors (IPA_INPUTS); outputs:
        list of pinned host tensors [B, L, H, F].  Work starts after what is
        already queued on `stream` (default: current) and `stream` waits for
        the last result at the end."""
        caller = stream if stream is not None else torch.cuda.current_stream(self.device)
        start = torch.cuda.Event()
        start.record(caller)
        for st in (self.up, self.comp, self.down):
            st.wait_event(start)
        p = self.plan.params
        for k, (inp, out_host) in enumerate(zip(inputs, outputs)):
            s = k % 2
            with torch.cuda.stream(self.up):
                self.up.wait_event(self.consumed[s])         # call k-2 has read staging set s
                dev = self._stage(s, inp)
                self.uploaded[s].record(self.up)
            with torch.cuda.stream(self.comp):
                self.comp.wait_event(self.uploaded[s])
                self.comp.wait_event(self.downloaded[s])     # call k-2's result has left buffer s
                if self.outs[s] is None:
                    self.outs[s] = torch.empty((p.B, p.L, p.H, self.plan.F), dtype=torch.float32,
                                               device=self.device)
                self.plan.prologue(*[dev[n] for n in IPA_INPUTS])
                self.consumed[s].record(self.comp)
                self.plan.core(self.outs[s])
                self.computed[s].record(self.comp)
            with torch.cuda.stream(self.down):
                self.down.wait_event(self.computed[s])
                out_host.copy_(self.outs[s], non_blocking=True)
                self.downloaded[s].record(self.down)
        end = torch.cuda.Event()
        end.record(self.down)
        caller.wait_event(end)
        return outputs


# ------------------------------------------------------------------ variant
GEO_INPUTS = ("q_direction", "k_direction", "q_point", "k_point", "values", "direction_scale",
              "distance_scale", "output_weight", "output_bias", "rotation", "translation",
              "frame_mask", "pair_mask")


class GeoPlan:
    def __init__(self, B, N, H, M, Cout, device="cuda"):
        self.params = GeoParams(B, N, H, M, Cout)
        nbytes = int(library().geo_attn_workspace_size(ctypes.byref(self.params)))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, inp: dict, *, with_attention: bool = True, out: Optional[dict] = None, stream=None):
        p = self.params
        dev = inp["q_direction"].device
        _require_cuda(*[inp.get(n) for n in GEO_INPUTS])
        if out is None:
            out = {"vectors": torch.empty((p.B, p.N, p.H, p.M, 3), dtype=torch.float32, device=dev),
                   "output": torch.empty((p.B, p.N, p.Cout), dtype=torch.float32, device=dev),
                   "attention": (torch.empty((p.B, p.H, p.N, p.N), dtype=torch.float32, device=dev)
                                 if with_attention else None)}
        pm = inp.get("pair_mask")
        if pm is not None and pm.dim() == 4 and tuple(pm.shape) != (p.B, p.H, p.N, p.N):
            pm = pm.expand(p.B, p.H, p.N, p.N)
        descs = [tensor_desc(inp.get(n)) for n in GEO_INPUTS[:-1]] + [tensor_desc(pm)]
        descs += [tensor_desc(out["vectors"]), tensor_desc(out["output"]), tensor_desc(out.get("attention"))]
        st = library().geo_attn_fwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                    ctypes.c_void_p(self.workspace.data_ptr()),
                                    ctypes.c_size_t(self.workspace.numel()),
                                    ctypes.c_void_p(_stream_ptr(stream)),
                                    ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def check(self):
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


def geo_attn(inp: dict, *, with_attention: bool = True, stream=None, check: bool = True):
    B, N, H, _ = inp["q_direction"].shape
    M = inp["values"].shape[3]
    Cout = inp["output_weight"].shape[1]
    plan = GeoPlan(B, N, H, M, Cout, device=inp["q_direction"].device)
    res = plan(inp, with_attention=with_attention, stream=stream)
    if check:
        plan.check()
    return res


class GeoGradPlan:
    """Gradients of the variant (Required behavior: the operator is
    differentiated, zero distance derivative at a zero displacement); the
    workspace is owned by the plan and reused across calls of one shape."""

    def __init__(self, B, N, H, M, Cout, device="cuda"):
        self.params = GeoParams(B, N, H, M, Cout)
        nbytes = int(library().geo_attn_bwd_workspace_size(ctypes.byref(self.params)))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, inp: dict, g_output, g_attention=None, g_vectors=None, *, out: Optional[dict] = None,
                 stream=None):
        p = self.params
        dev = inp["q_direction"].device
        _require_cuda(*[inp.get(n) for n in GEO_INPUTS], g_output, g_attention, g_vectors)
        if out is None:
            out = {n: (torch.empty(tuple(inp[n].shape), dtype=torch.float32, device=dev)
                       if inp.get(n) is not None else None) for n in GEO_GRADS}
        pm = inp.get("pair_mask")
        if pm is not None and pm.dim() == 4 and tuple(pm.shape) != (p.B, p.H, p.N, p.N):
            pm = pm.expand(p.B, p.H, p.N, p.N)
        descs = [tensor_desc(inp.get(n)) for n in GEO_INPUTS[:-1]] + [tensor_desc(pm)]
        descs += [tensor_desc(g_output), tensor_desc(g_attention), tensor_desc(g_vectors)]
        grads = GeoGrads(*[tensor_desc(out.get(n)) for n in GEO_GRADS])
        st = library().geo_attn_bwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs], ctypes.byref(grads),
                                    ctypes.c_void_p(self.workspace.data_ptr()),
                                    ctypes.c_size_t(self.workspace.numel()),
                                    ctypes.c_void_p(_stream_ptr(stream)),
                                    ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def check(self):
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


def geo_attn_backward(inp: dict, g_output, g_attention=None, g_vectors=None, *, stream=None,
                      check: bool = True) -> dict:
    """Gradients of sum(g_output * output) + sum(g_attention * attention)
    + sum(g_vectors * vectors) with respect to every floating input (fp32)."""
    B, N, H, _ = inp["q_direction"].shape
    M = inp["values"].shape[3]
    Cout = inp["output_weight"].shape[1]
    plan = GeoGradPlan(B, N, H, M, Cout, device=inp["q_direction"].device)
    res = plan(inp, g_output, g_attention, g_vectors, stream=stream)
    if check:
        plan.check()
    return res


# ------------------------------------------------------------------ MEET
MEET_INPUTS = ("q", "k", "v", "x", "rho", "s", "mask")


class MeetPlan:
    """Distance-aware attention of MEET (§2.2, eq. (6)) on the fused core:
    workspace owned by the plan, reused across calls of the same shape."""

    def __init__(self, B: int, L: int, H: int, C: int = 16, device="cuda"):
        self.params = MeetParams(B, L, H, C)
        nbytes = int(library().meet_attn_workspace_size(ctypes.byref(self.params)))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope (C must be 16)")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, q, k, v, x, rho, s, mask, out=None, stream=None):
        p = self.params
        _require_cuda(q, k, v, x, rho, s, mask)
        if out is None:
            out = torch.empty((p.B, p.L, p.H, p.C), dtype=torch.float32, device=q.device)
        descs = [tensor_desc(t) for t in (q, k, v, x, rho, s, mask, out)]
        st = library().meet_attn_fwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                     ctypes.c_void_p(self.workspace.data_ptr()),
                                     ctypes.c_size_t(self.workspace.numel()),
                                     ctypes.c_void_p(_stream_ptr(stream)),
                                     ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def check(self):
        """Raise if a device-side bounded wait expired (call after a sync)."""
        v = int(self.dev_err.item())
        if v != 0:
            st = library().ipa_device_error_status(v)
            raise IpaError(st, f"device error word {v}")


def meet_attn(inp: dict, *, out=None, stream=None, check: bool = True):
    """One call of the distance-aware attention on CUDA tensors `inp`
    (keys MEET_INPUTS); returns o [B, L, H, C]."""
    B, L, H, C = inp["q"].shape
    plan = MeetPlan(B, L, H, C, device=inp["q"].device)
    res = plan(*[inp[n] for n in MEET_INPUTS], out=out, stream=stream)
    if check:
        torch.cuda.synchronize()
        plan.check()
    return res


# ------------------------------------------------------------------ frames
def frames_from_backbone(n, ca, c, rot=None, trans=None, stream=None):
    """Residue frames (rot [B, L, 3, 3], trans [B, L, 3]) from backbone atoms
    n, ca, c [B, L, 3] on the GPU (Gram-Schmidt on C_alpha)."""
    _require_cuda(n, ca, c)
    B, L = n.shape[0], n.shape[1]
    if rot is None:
        rot = torch.empty((B, L, 3, 3), dtype=torch.float32, device=n.device)
    if trans is None:
        trans = torch.empty((B, L, 3), dtype=torch.float32, device=n.device)
    descs = [tensor_desc(t) for t in (n, ca, c, rot, trans)]
    st = library().ipa_frames_from_backbone(B, L, *[ctypes.byref(d) for d in descs],
                                            ctypes.c_void_p(_stream_ptr(stream)))
    if st != 0:
        raise IpaError(st, library().ipa_status_string(st).decode())
    return rot, trans


# ------------------------------------------------------------------ distogram
def knn_distogram(x, mask, k: int, edges, *, stream=None):
    """Local nearest-neighbour distogram of positions x [B, L, 3] (CUDA
    tensors): (idx [B, L, k] int32, bins [B, L, k] int32, hist [B, L, nb]
    float32), nb = len(edges) + 1; `edges` is a host sequence of increasing
    distances (Angstrom)."""
    _require_cuda(x, mask)
    B, L = x.shape[0], x.shape[1]
    e = (ctypes.c_float * max(1, len(edges)))(*[float(v) for v in edges])
    idx = torch.empty((B, L, k), dtype=torch.int32, device=x.device)
    bins = torch.empty((B, L, k), dtype=torch.int32, device=x.device)
    hist = torch.empty((B, L, len(edges) + 1), dtype=torch.float32, device=x.device)
    descs = [tensor_desc(t) for t in (x, mask)]
    outs = [tensor_desc(t) for t in (idx, bins, hist)]
    st = library().ipa_knn_distogram(B, L, k, len(edges), *[ctypes.byref(d) for d in descs], e,
                                     *[ctypes.byref(d) for d in outs], ctypes.c_void_p(_stream_ptr(stream)))
    if st != 0:
        raise IpaError(st, library().ipa_status_string(st).decode())
    return idx, bins, hist


# ------------------------------------------------------------------ projections
class LinearPlan:
    """y = x W + b on the tensor cores (fp16 operands, fp32 accumulation);
    the plan owns the workspace for one (M, K, N)."""

    def __init__(self, M: int, K: int, N: int, device="cuda"):
        self.M, self.K, self.N = M, K, N
        nbytes = int(library().ipa_linear_workspace_size(M, K, N))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, x, w, b=None, *, out=None, stream=None):
        _require_cuda(x, w, b)
        if out is None:
            out = torch.empty((self.M, self.N), dtype=torch.float32, device=x.device)
        descs = [tensor_desc(t) for t in (x, w, b, out)]
        st = library().ipa_linear_fwd(self.M, self.K, self.N, *[ctypes.byref(d) for d in descs],
                                      ctypes.c_void_p(self.workspace.data_ptr()),
                                      ctypes.c_size_t(self.workspace.numel()),
                                      ctypes.c_void_p(_stream_ptr(stream)),
                                      ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def check(self):
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


def linear(x, w, b=None, *, stream=None, check: bool = True):
    """y = x W + b for x [M, K], W [K, N] (fp32 tensors on the GPU)."""
    plan = LinearPlan(x.shape[0], x.shape[1], w.shape[1], device=x.device)
    y = plan(x, w, b, stream=stream)
    if check:
        plan.check()
    return y


# ------------------------------------------------------------------ IPA layer
MODULE_INPUTS = ("s", "rot", "trans", "z1", "z2", "w_bias", "gamma", "mask", "w_in", "b_in", "w_out", "b_out")


class ModulePlan:
    """The IPA layer around the core: input projection to q, k, v and the
    local points, the fused core, output projection (one C-ABI call)."""

    def __init__(self, B, L, H, C, Pq, Pv, R, Cz, c_s, device="cuda", **consts):
        self.params = ModuleParams(ipa_params(B, L, H, C, Pq, Pv, R, Cz, **consts), c_s)
        nbytes = int(library().ipa_module_workspace_size(ctypes.byref(self.params)))
        if nbytes == 0:
            raise IpaError(6, "dimensions outside the supported envelope")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=device)
        self.F = C + 4 * Pv + Cz

    def __call__(self, inp: dict, *, out=None, core_out=None, stream=None):
        p = self.params
        _require_cuda(*[inp.get(n) for n in MODULE_INPUTS], core_out)
        if out is None:
            out = torch.empty((p.core.B, p.core.L, p.c_s), dtype=torch.float32, device=inp["s"].device)
        descs = [tensor_desc(inp.get(n)) for n in MODULE_INPUTS] + [tensor_desc(out), tensor_desc(core_out)]
        st = library().ipa_module_fwd(ctypes.byref(p), *[ctypes.byref(d) for d in descs],
                                      ctypes.c_void_p(self.workspace.data_ptr()),
                                      ctypes.c_size_t(self.workspace.numel()),
                                      ctypes.c_void_p(_stream_ptr(stream)),
                                      ctypes.c_void_p(self.dev_err.data_ptr()))
        if st != 0:
            raise IpaError(st, library().ipa_status_string(st).decode())
        return out

    def check(self):
        v = int(self.dev_err.item())
        if v != 0:
            self.dev_err.zero_()
            raise IpaError(int(library().ipa_device_error_status(v)), f"device error code {v}")


def ipa_module(inp: dict, *, with_core: bool = False, stream=None, check: bool = True, **consts):
    """IPA layer forward; with_core also returns the core output [B, L, H, F]."""
    B, L, c_s = inp["s"].shape
    H = inp["gamma"].shape[0]
    z1 = inp["z1"]
    R, Cz = z1.shape[2], z1.shape[3]
    width = inp["w_in"].shape[1]
    per_head = width // H                      # 3 C + 3 (2 Pq + Pv) with C = 16, Pq = 4, Pv = 8 supported
    C, Pq, Pv = 16, 4, 8
    if per_head != 3 * C + 3 * (2 * Pq + Pv):
        raise IpaError(6, "the core supports C = 16, Pq = 4, Pv = 8")
    plan = ModulePlan(B, L, H, C, Pq, Pv, R, Cz, c_s, device=inp["s"].device, **consts)
    core = (torch.empty((B, L, H, plan.F), dtype=torch.float32, device=inp["s"].device) if with_core else None)
    out = plan(inp, core_out=core, stream=stream)
    if check:
        plan.check()
    return (out, core) if with_core else out
