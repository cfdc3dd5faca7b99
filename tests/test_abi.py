"""CPU-only checks of the C ABI boundary: the library loads, exports every
function include/flashipa_b200.h declares, and rejects bad arguments before
launching anything.  No test here runs device code."""
import ctypes
import os
import re

import numpy as np
import pytest

from rna_structure_models_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashipa_b200.h")

FAKE = 1 << 20  # a non-null, 256-aligned address that is never dereferenced


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"IPA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    assert {"ipa_attn_fwd", "ipa_attn_workspace_size", "geo_attn_fwd", "geo_attn_workspace_size",
            "ipa_status_string"} <= names


def test_library_exports_every_declared_symbol():
    lib = api.library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(api.EXPORTED) == set(declared_functions())


def test_status_strings_and_version():
    lib = api.library()
    for code in range(10):
        assert lib.ipa_status_string(code) != b"unknown status"
    assert b"sm_100a" in lib.ipa_version()
    assert not lib.ipa_version().endswith(b"bounds-checked")   # the product build carries no checks
    assert lib.ipa_device_error_status(0) == 0
    assert lib.ipa_device_error_status(1) == 8       # bounded wait expired -> IPA_ERR_TIMEOUT
    assert lib.ipa_device_error_status(7) == 7
    # bounds-checked build: 0x10000 | file tag << 12 | source line -> IPA_ERR_BOUNDS
    assert lib.ipa_device_error_status(0x10000 | (11 << 12) | 873) == 9


def test_checked_build_exports_the_same_symbols_and_reports_itself():
    from rna_structure_models_b200 import build
    if build.checked_is_stale():
        pytest.skip("bounds-checked library not built (python -m rna_structure_models_b200.build)")
    chk = ctypes.CDLL(build.CHECKED_LIB)
    chk.ipa_version.restype = ctypes.c_char_p
    assert chk.ipa_version().endswith(b"bounds-checked")
    for name in api.EXPORTED:
        assert hasattr(chk, name), name


def desc(shape, dtype=api.IPA_DTYPE_F32, ptr=FAKE, strides=None):
    d = api.IpaTensor()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.size[i] = s
        d.stride[i] = st
    return d


def ipa_args(B=1, L=64, H=4, C=16, Pq=4, Pv=8, R=2, Cz=16, **over):
    F = C + 4 * Pv + Cz
    shapes = {"q": (B, L, H, C), "k": (B, L, H, C), "v": (B, L, H, C),
              "q_pts": (B, L, H, Pq, 3), "k_pts": (B, L, H, Pq, 3), "v_pts": (B, L, H, Pv, 3),
              "rot": (B, L, 3, 3), "trans": (B, L, 3), "z1": (B, L, R, Cz), "z2": (B, L, R, Cz),
              "w_bias": (Cz, H), "gamma": (H,), "mask": (B, L), "out": (B, L, H, F)}
    ds = {k: desc(s, api.IPA_DTYPE_BOOL if k == "mask" else api.IPA_DTYPE_F32) for k, s in shapes.items()}
    ds.update(over)
    return api.ipa_params(B, L, H, C, Pq, Pv, R, Cz), ds


ORDER = ("q", "k", "v", "q_pts", "k_pts", "v_pts", "rot", "trans", "z1", "z2", "w_bias", "gamma",
         "mask", "out")


def call_ipa(p, ds, ws_bytes=None, ws_ptr=FAKE):
    lib = api.library()
    if ws_bytes is None:
        ws_bytes = lib.ipa_attn_workspace_size(ctypes.byref(p))
    return lib.ipa_attn_fwd(ctypes.byref(p), *[ctypes.byref(ds[k]) if ds[k] is not None else None
                                               for k in ORDER],
                            ctypes.c_void_p(ws_ptr), ctypes.c_size_t(ws_bytes), None,
                            ctypes.c_void_p(FAKE))


def test_workspace_size_is_linear_in_L_and_zero_when_invalid():
    lib = api.library()
    sizes = []
    for L in (2048, 4096, 8192, 16384):
        p = api.ipa_params(1, L, 12, 16, 4, 8, 2, 128)
        sizes.append(lib.ipa_attn_workspace_size(ctypes.byref(p)))
    Ls = np.array([2048, 4096, 8192, 16384], float)
    marg = np.diff(np.array(sizes, float)) / np.diff(Ls)     # bytes per added residue
    assert marg.max() / marg.min() < 1.01, marg
    # the rest is a constant: the core's key-split reserve (two chunks of
    # partial accumulators per resident CTA pair), bounded whatever L is
    const = sizes[0] - marg[0] * Ls[0]
    assert 0 < const < 64 * 2 ** 20, const
    bad = api.ipa_params(1, 64, 4, 32, 4, 8, 2, 16)      # C = 32 is outside the envelope
    assert lib.ipa_attn_workspace_size(ctypes.byref(bad)) == 0


@pytest.mark.parametrize("case,expect", [
    ("null_tensor", 1), ("shape", 2), ("neg_stride", 3), ("dtype", 4), ("workspace", 5),
    ("ws_align", 5), ("unsupported", 6), ("mask_dtype", 4), ("out_noncontig", 3), ("null_params", 1),
])
def test_ipa_rejects_bad_arguments_before_launch(case, expect):
    p, ds = ipa_args()
    ws = None
    ws_ptr = FAKE
    if case == "null_tensor":
        ds["k"] = desc((1, 64, 4, 16), ptr=None)
    elif case == "shape":
        ds["v"] = desc((1, 63, 4, 16))
    elif case == "neg_stride":
        ds["q"] = desc((1, 64, 4, 16), strides=(4096, 64, -16, 1))
    elif case == "dtype":
        ds["z1"] = desc((1, 64, 2, 16), dtype=api.IPA_DTYPE_F64)
    elif case == "workspace":
        ws = 1024
    elif case == "ws_align":
        ws_ptr = FAKE + 8
    elif case == "unsupported":
        p, ds = ipa_args(Pv=4)
    elif case == "mask_dtype":
        ds["mask"] = desc((1, 64), dtype=api.IPA_DTYPE_F32)
    elif case == "out_noncontig":
        ds["out"] = desc((1, 64, 4, 64), strides=(64 * 4 * 128, 4 * 128, 128, 1))
    if case == "null_params":
        lib = api.library()
        st = lib.ipa_attn_fwd(None, *[ctypes.byref(ds[k]) for k in ORDER], ctypes.c_void_p(FAKE),
                              ctypes.c_size_t(1 << 30), None, ctypes.c_void_p(FAKE))
    else:
        st = call_ipa(p, ds, ws, ws_ptr)
    assert st == expect


def geo_args(B=1, N=32, H=2, M=2, Cout=8, dt=api.IPA_DTYPE_F32, **over):
    shapes = {"q_direction": (B, N, H, 3), "k_direction": (B, N, H, 3), "q_point": (B, N, H, 3),
              "k_point": (B, N, H, 3), "values": (B, N, H, M, 3), "direction_scale": (H,),
              "distance_scale": (H,), "output_weight": (H * M * 3, Cout), "output_bias": (Cout,),
              "rotation": (B, N, 3, 3), "translation": (B, N, 3)}
    ds = {k: desc(s, dt) for k, s in shapes.items()}
    ds["frame_mask"] = desc((B, N), api.IPA_DTYPE_BOOL)
    ds["pair_mask"] = desc((B, H, N, N), api.IPA_DTYPE_BOOL)
    ds["out_vectors"] = desc((B, N, H, M, 3))
    ds["out_output"] = desc((B, N, Cout))
    ds["out_attention"] = desc((B, H, N, N))
    ds.update(over)
    return api.GeoParams(B, N, H, M, Cout), ds


GEO_ORDER = api.GEO_INPUTS + ("out_vectors", "out_output", "out_attention")


def call_geo(p, ds, ws_bytes=None):
    lib = api.library()
    if ws_bytes is None:
        ws_bytes = lib.geo_attn_workspace_size(ctypes.byref(p))
    return lib.geo_attn_fwd(ctypes.byref(p), *[ctypes.byref(ds[k]) if ds[k] is not None else None
                                               for k in GEO_ORDER],
                            ctypes.c_void_p(FAKE), ctypes.c_size_t(ws_bytes), None, ctypes.c_void_p(FAKE))


@pytest.mark.parametrize("case,expect", [
    ("mixed_dtype", 4), ("pair_mask_shape", 2), ("values_shape", 2), ("workspace", 5),
    ("too_many_channels", 6), ("frame_mask_dtype", 4), ("att_noncontig", 3),
])
def test_geo_rejects_bad_arguments_before_launch(case, expect):
    p, ds = geo_args()
    ws = None
    if case == "mixed_dtype":
        ds["k_point"] = desc((1, 32, 2, 3), api.IPA_DTYPE_F64)
    elif case == "pair_mask_shape":
        ds["pair_mask"] = desc((1, 2, 32, 31), api.IPA_DTYPE_BOOL)
    elif case == "values_shape":
        ds["values"] = desc((1, 32, 2, 3, 3))
    elif case == "workspace":
        ws = 100
    elif case == "too_many_channels":
        p, ds = geo_args(H=40, M=4)
    elif case == "frame_mask_dtype":
        ds["frame_mask"] = desc((1, 32))
    elif case == "att_noncontig":
        ds["out_attention"] = desc((1, 2, 32, 32), strides=(4096, 2048, 64, 1))
    assert call_geo(p, ds, ws) == expect


def test_package_import_does_not_load_the_library():
    import importlib
    import subprocess
    import sys
    code = ("import rna_structure_models_b200, rna_structure_models_b200.synth, sys;"
            "print(any('libflashipa' in l for l in open('/proc/self/maps')))")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert out.stdout.strip() == "False", out.stderr
    importlib.import_module("rna_structure_models_b200")


def meet_call(B=2, L=64, H=3, C=16, ws_bytes=None, ws_ptr=FAKE, **over):
    lib = api.library()
    p = api.MeetParams(B, L, H, C)
    shapes = {"q": (B, L, H, C), "k": (B, L, H, C), "v": (B, L, H, C), "x": (B, L, 3), "rho": (H,), "s": (H,),
              "mask": (B, L), "out": (B, L, H, C)}
    ds = {k: desc(sh, api.IPA_DTYPE_BOOL if k == "mask" else api.IPA_DTYPE_F32) for k, sh in shapes.items()}
    ds.update(over)
    if ws_bytes is None:
        ws_bytes = lib.meet_attn_workspace_size(ctypes.byref(p))
    return lib.meet_attn_fwd(ctypes.byref(p), *[ctypes.byref(ds[k]) for k in api.MEET_INPUTS + ("out",)],
                             ctypes.c_void_p(ws_ptr), ctypes.c_size_t(ws_bytes), None, ctypes.c_void_p(FAKE))


def test_meet_workspace_linear_in_L_and_zero_outside_envelope():
    lib = api.library()
    per = []
    for L in (2048, 4096, 8192):
        per.append(lib.meet_attn_workspace_size(ctypes.byref(api.MeetParams(1, L, 8, 16))) / L)
    assert max(per) / min(per) < 1.01
    assert lib.meet_attn_workspace_size(ctypes.byref(api.MeetParams(1, 64, 8, 32))) == 0   # C must be 16


@pytest.mark.parametrize("case,expect", [
    ("unsupported_C", 6), ("shape_x", 2), ("dtype_mask", 4), ("null_rho", 1), ("workspace", 5),
    ("out_noncontig", 3),
])
def test_meet_rejects_bad_arguments_before_launch(case, expect):
    if case == "unsupported_C":
        assert meet_call(C=32, ws_bytes=1 << 30) == expect
        return
    over, ws_bytes = {}, None
    if case == "shape_x":
        over["x"] = desc((2, 64, 4))
    elif case == "dtype_mask":
        over["mask"] = desc((2, 64), api.IPA_DTYPE_F32)
    elif case == "null_rho":
        over["rho"] = desc((3,), ptr=None)
    elif case == "workspace":
        ws_bytes = 1024
    elif case == "out_noncontig":
        over["out"] = desc((2, 64, 3, 16), strides=(64 * 3 * 16, 1, 64, 3 * 64))
    assert meet_call(ws_bytes=ws_bytes, **over) == expect


def frames_call(B=2, L=64, **over):
    lib = api.library()
    ds = {"n": desc((B, L, 3)), "ca": desc((B, L, 3)), "c": desc((B, L, 3)),
          "rot": desc((B, L, 3, 3)), "trans": desc((B, L, 3))}
    ds.update(over)
    return lib.ipa_frames_from_backbone(B, L, *[ctypes.byref(ds[k]) for k in ("n", "ca", "c", "rot", "trans")],
                                        ctypes.c_void_p(FAKE))


@pytest.mark.parametrize("case,expect", [
    ("empty", 2), ("shape_ca", 2), ("dtype_c", 4), ("null_n", 1), ("rot_noncontig", 3), ("trans_shape", 2),
])
def test_frames_rejects_bad_arguments_before_launch(case, expect):
    if case == "empty":
        assert frames_call(B=0) == expect
        return
    over = {}
    if case == "shape_ca":
        over["ca"] = desc((2, 63, 3))
    elif case == "dtype_c":
        over["c"] = desc((2, 64, 3), api.IPA_DTYPE_BOOL)
    elif case == "null_n":
        over["n"] = desc((2, 64, 3), ptr=None)
    elif case == "rot_noncontig":
        over["rot"] = desc((2, 64, 3, 3), strides=(576, 9, 1, 3))
    elif case == "trans_shape":
        over["trans"] = desc((2, 64, 4))
    assert frames_call(**over) == expect


def geo_bwd_call(p, ds, grads_over=None, ws_bytes=None, **up_over):
    lib = api.library()
    B, N, H, M, Cout = p.B, p.N, p.H, p.M, p.Cout
    up = {"g_output": desc((B, N, Cout)), "g_attention": desc((B, H, N, N)), "g_vectors": desc((B, N, H, M, 3))}
    up.update(up_over)
    shapes = {"q_direction": (B, N, H, 3), "k_direction": (B, N, H, 3), "q_point": (B, N, H, 3),
              "k_point": (B, N, H, 3), "values": (B, N, H, M, 3), "direction_scale": (H,),
              "distance_scale": (H,), "output_weight": (H * M * 3, Cout), "output_bias": (Cout,),
              "rotation": (B, N, 3, 3), "translation": (B, N, 3)}
    gd = {k: desc(s) for k, s in shapes.items()}
    gd.update(grads_over or {})
    grads = api.GeoGrads(*[gd[k] for k in api.GEO_GRADS])
    if ws_bytes is None:
        ws_bytes = lib.geo_attn_bwd_workspace_size(ctypes.byref(p))
    return lib.geo_attn_bwd(ctypes.byref(p), *[ctypes.byref(ds[k]) if ds[k] is not None else None
                                               for k in api.GEO_INPUTS],
                            *[ctypes.byref(up[k]) if up[k] is not None else None
                              for k in ("g_output", "g_attention", "g_vectors")],
                            ctypes.byref(grads), ctypes.c_void_p(FAKE), ctypes.c_size_t(ws_bytes),
                            ctypes.c_void_p(FAKE), None)


def test_geo_bwd_workspace_grows_with_the_problem_and_is_zero_outside_envelope():
    lib = api.library()
    small = lib.geo_attn_bwd_workspace_size(ctypes.byref(api.GeoParams(1, 256, 8, 4, 256)))
    big = lib.geo_attn_bwd_workspace_size(ctypes.byref(api.GeoParams(2, 2048, 8, 4, 256)))
    assert 0 < small < big
    assert big > lib.geo_attn_workspace_size(ctypes.byref(api.GeoParams(2, 2048, 8, 4, 256)))
    assert lib.geo_attn_bwd_workspace_size(ctypes.byref(api.GeoParams(1, 64, 40, 4, 8))) == 0


@pytest.mark.parametrize("case,expect", [
    ("g_output_shape", 2), ("g_att_dtype", 4), ("grad_noncontig", 3), ("bias_grad_missing", 1),
    ("bias_grad_without_bias", 2), ("workspace", 5), ("input_shape", 2),
])
def test_geo_bwd_rejects_bad_arguments_before_launch(case, expect):
    p, ds = geo_args()
    grads_over, up, ws = {}, {}, None
    if case == "g_output_shape":
        up["g_output"] = desc((1, 32, 7))
    elif case == "g_att_dtype":
        up["g_attention"] = desc((1, 2, 32, 32), api.IPA_DTYPE_F64)
    elif case == "grad_noncontig":
        grads_over["values"] = desc((1, 32, 2, 2, 3), strides=(384, 12, 6, 1, 2))
    elif case == "bias_grad_missing":
        grads_over["output_bias"] = desc((8,), ptr=None)
    elif case == "bias_grad_without_bias":
        ds["output_bias"] = desc((8,), ptr=None)
    elif case == "workspace":
        ws = 4096
    elif case == "input_shape":
        ds["translation"] = desc((1, 32, 4))
    assert geo_bwd_call(p, ds, grads_over, ws, **up) == expect



@pytest.mark.parametrize("case,expect", [
    ("shape_w", 2), ("dtype_x", 4), ("y_noncontig", 3), ("bias_shape", 2), ("workspace", 5), ("big_k", 6),
    ("zero_m", 2),
])
def test_linear_rejects_bad_arguments_before_launch(case, expect):
    lib = api.library()
    M, K, N = 200, 96, 70
    ds = {"x": desc((M, K)), "w": desc((K, N)), "b": desc((N,)), "y": desc((M, N))}
    ws = None
    if case == "shape_w":
        ds["w"] = desc((K + 1, N))
    elif case == "dtype_x":
        ds["x"] = desc((M, K), api.IPA_DTYPE_F64)
    elif case == "y_noncontig":
        ds["y"] = desc((M, N), strides=(1, M))
    elif case == "bias_shape":
        ds["b"] = desc((N + 1,))
    elif case == "workspace":
        ws = 512
    elif case == "big_k":
        K = 70000
        ds["x"], ds["w"] = desc((M, K)), desc((K, N))
        ws = 1 << 30
    elif case == "zero_m":
        M = 0
    if ws is None:
        ws = lib.ipa_linear_workspace_size(max(M, 1), K, N)
    st = lib.ipa_linear_fwd(M, K, N, *[ctypes.byref(ds[k]) for k in ("x", "w", "b", "y")],
                            ctypes.c_void_p(FAKE), ctypes.c_size_t(ws), None, None)
    assert st == expect


def test_linear_workspace_holds_both_fp16_operands():
    lib = api.library()
    assert lib.ipa_linear_workspace_size(4096, 384, 1152) >= 2 * (4096 + 1152) * 384
    assert lib.ipa_linear_workspace_size(10, 70000, 10) == 0


@pytest.mark.parametrize("case,expect", [
    ("s_rows_not_flat", 3), ("w_in_shape", 2), ("out_noncontig", 3), ("workspace", 5), ("core_C", 6),
    ("c_s_zero", 2), ("core_out_shape", 2), ("rot_shape", 2), ("mask_dtype", 4),
])
def test_module_rejects_bad_arguments_before_launch(case, expect):
    lib = api.library()
    B, L, H, Cz, cs = 2, 64, 3, 32, 40
    C, Pq, Pv, R = 16, 4, 8, 2
    width, F = H * (3 * C + 3 * (2 * Pq + Pv)), C + 4 * Pv + Cz
    p = api.ModuleParams(api.ipa_params(B, L, H, C, Pq, Pv, R, Cz), cs)
    ds = {"s": desc((B, L, cs)), "rot": desc((B, L, 3, 3)), "trans": desc((B, L, 3)), "z1": desc((B, L, R, Cz)),
          "z2": desc((B, L, R, Cz)), "w_bias": desc((Cz, H)), "gamma": desc((H,)),
          "mask": desc((B, L), api.IPA_DTYPE_BOOL), "w_in": desc((cs, width)), "b_in": desc((width,)),
          "w_out": desc((H * F, cs)), "b_out": desc((cs,)), "out": desc((B, L, cs)), "core_out": None}
    ws = None
    if case == "s_rows_not_flat":
        ds["s"] = desc((B, L, cs), strides=(L * cs + 8, cs, 1))
    elif case == "w_in_shape":
        ds["w_in"] = desc((cs, width + 1))
    elif case == "out_noncontig":
        ds["out"] = desc((B, L, cs), strides=(L * cs, 1, L))
    elif case == "workspace":
        ws = 1 << 10
    elif case == "core_C":
        p = api.ModuleParams(api.ipa_params(B, L, H, 32, Pq, Pv, R, Cz), cs)
        ws = 1 << 30
    elif case == "c_s_zero":
        p = api.ModuleParams(api.ipa_params(B, L, H, C, Pq, Pv, R, Cz), 0)
        ws = 1 << 30
    elif case == "core_out_shape":
        ds["core_out"] = desc((B, L, H, F + 1))
    elif case == "rot_shape":
        ds["rot"] = desc((B, L, 3, 4))
    elif case == "mask_dtype":
        ds["mask"] = desc((B, L))
    if ws is None:
        ws = lib.ipa_module_workspace_size(ctypes.byref(p))
    order = api.MODULE_INPUTS + ("out", "core_out")
    st = lib.ipa_module_fwd(ctypes.byref(p), *[ctypes.byref(ds[k]) if ds[k] is not None else None for k in order],
                            ctypes.c_void_p(FAKE), ctypes.c_size_t(ws), None, None)
    assert st == expect


def ipa_bwd_call(p, ds, extra, grads, ws_bytes=None, ws_ptr=FAKE):
    lib = api.library()
    if ws_bytes is None:
        ws_bytes = lib.ipa_attn_bwd_workspace_size(ctypes.byref(p))
    gs = api.IpaGrads(*[grads[n] for n in api.IPA_GRADS])
    return lib.ipa_attn_bwd(ctypes.byref(p), *[ctypes.byref(ds[k]) for k in ORDER],
                            *[ctypes.byref(extra[k]) if extra[k] is not None else None
                              for k in ("lse", "u_agg", "g_out")],
                            ctypes.byref(gs), ctypes.c_void_p(ws_ptr), ctypes.c_size_t(ws_bytes), None,
                            ctypes.c_void_p(FAKE))


def bwd_args(B=1, L=64, H=4, R=2, Cz=16):
    p, ds = ipa_args(B=B, L=L, H=H, R=R, Cz=Cz)
    F = 16 + 32 + Cz
    extra = {"lse": desc((B, H, L)), "u_agg": desc((B, L, H, R, Cz)), "g_out": desc((B, L, H, F))}
    grads = {n: desc(tuple(ds[n].size[i] for i in range(ds[n].ndim))) for n in api.IPA_GRADS}
    return p, ds, extra, grads


def test_bwd_workspace_is_linear_in_L_and_zero_when_invalid():
    lib = api.library()
    sizes = []
    for L in (2048, 4096, 8192, 16384):
        p = api.ipa_params(1, L, 12, 16, 4, 8, 2, 128)
        sizes.append(lib.ipa_attn_bwd_workspace_size(ctypes.byref(p)))
        assert lib.ipa_attn_bwd_workspace_size(ctypes.byref(p)) > lib.ipa_attn_workspace_size(ctypes.byref(p))
    Ls = np.array([2048, 4096, 8192, 16384], float)
    marg = np.diff(np.array(sizes, float)) / np.diff(Ls)     # bytes per added residue
    assert marg.max() / marg.min() < 1.02, marg
    # plus a bounded constant: the key pass's split reserve (one round of
    # chunks on the resident CTAs) and the per-block reduction rounding
    const = sizes[0] - marg[0] * Ls[0]
    assert abs(const) < 64 * 2 ** 20, const
    bad = api.ipa_params(1, 64, 4, 16, 4, 8, 2, 20)      # Cz not a multiple of 16
    assert lib.ipa_attn_bwd_workspace_size(ctypes.byref(bad)) == 0


@pytest.mark.parametrize("case,expect", [
    ("ok_shape_check_only", None), ("null_grads", 1), ("lse_shape", 2), ("uagg_dtype", 4), ("g_out_shape", 2),
    ("grad_noncontig", 3), ("grad_shape", 2), ("workspace", 5), ("ws_align", 5), ("unsupported", 6),
])
def test_ipa_bwd_rejects_bad_arguments_before_launch(case, expect):
    p, ds, extra, grads = bwd_args()
    ws, ws_ptr = None, FAKE
    if case == "ok_shape_check_only":
        return                                   # a valid call would launch: nothing to run without a GPU
    if case == "null_grads":
        lib = api.library()
        st = lib.ipa_attn_bwd(ctypes.byref(p), *[ctypes.byref(ds[k]) for k in ORDER],
                              *[ctypes.byref(extra[k]) for k in ("lse", "u_agg", "g_out")], None,
                              ctypes.c_void_p(FAKE), ctypes.c_size_t(1 << 30), None, ctypes.c_void_p(FAKE))
        assert st == expect
        return
    if case == "lse_shape":
        extra["lse"] = desc((1, 64, 4))
    elif case == "uagg_dtype":
        extra["u_agg"] = desc((1, 64, 4, 2, 16), dtype=api.IPA_DTYPE_F64)
    elif case == "g_out_shape":
        extra["g_out"] = desc((1, 64, 4, 63))
    elif case == "grad_noncontig":
        grads["q"] = desc((1, 64, 4, 16), strides=(64 * 4 * 32, 4 * 32, 32, 1))
    elif case == "grad_shape":
        grads["z2"] = desc((1, 64, 2, 15))
    elif case == "workspace":
        ws = 1024
    elif case == "ws_align":
        ws_ptr = FAKE + 8
    elif case == "unsupported":
        p, ds, extra, grads = bwd_args()
        p.C = 32
    assert ipa_bwd_call(p, ds, extra, grads, ws, ws_ptr) == expect


@pytest.mark.parametrize("case,expect", [("lse_shape", 2), ("uagg_align", 3), ("null_lse", 1)])
def test_ipa_fwd_train_rejects_bad_outputs_before_launch(case, expect):
    p, ds = ipa_args()
    lse, uagg = desc((1, 4, 64)), desc((1, 64, 4, 2, 16))
    if case == "lse_shape":
        lse = desc((1, 64, 4))
    elif case == "uagg_align":
        uagg = desc((1, 64, 4, 2, 16), ptr=FAKE + 4)
    elif case == "null_lse":
        lse = desc((1, 4, 64), ptr=None)
    lib = api.library()
    ws = lib.ipa_attn_workspace_size(ctypes.byref(p))
    st = lib.ipa_attn_fwd_train(ctypes.byref(p), *[ctypes.byref(ds[k]) for k in ORDER], ctypes.byref(lse),
                                ctypes.byref(uagg), ctypes.c_void_p(FAKE), ctypes.c_size_t(ws), None,
                                ctypes.c_void_p(FAKE))
    assert st == expect


def test_packed_host_layout_matches_the_staging_order():
    # inputs in argument order, each at a multiple of 256 bytes, sized as the
    # dense fp32 (mask: one byte) tensors; the staging area holds them at the
    # same offsets, plus the result
    lib = api.library()
    p, ds = ipa_args(B=2, L=100, H=3, Cz=32)
    offs = (ctypes.c_size_t * 13)()
    n = lib.ipa_attn_host_packed_layout(ctypes.byref(p), ctypes.byref(offs))
    sizes = []
    for k in ORDER[:13]:
        cnt = 1
        for d in range(ds[k].ndim):
            cnt *= ds[k].size[d]
        sizes.append(cnt * (1 if k == "mask" else 4))
    o = list(offs)
    assert o[0] == 0 and all(x % 256 == 0 for x in o)
    for t in range(12):
        assert o[t + 1] == o[t] + (sizes[t] + 255) // 256 * 256
    assert n == o[12] + (sizes[12] + 255) // 256 * 256
    assert n < lib.ipa_attn_host_staging_size(ctypes.byref(p))
    bad = api.ipa_params(1, 64, 4, 32, 4, 8, 2, 16)          # C outside the envelope
    assert lib.ipa_attn_host_packed_layout(ctypes.byref(bad), ctypes.byref(offs)) == 0
    assert lib.ipa_attn_host_packed_layout(ctypes.byref(p), None) == 0


@pytest.mark.parametrize("case,expect", [("null_inputs", 1), ("short_buffer", 2), ("null_out", 1),
                                         ("out_shape", 2)])
def test_packed_host_call_rejects_bad_arguments_before_launch(case, expect):
    lib = api.library()
    p, ds = ipa_args()
    offs = (ctypes.c_size_t * 13)()
    n = lib.ipa_attn_host_packed_layout(ctypes.byref(p), ctypes.byref(offs))
    host, nbytes, out = ctypes.c_void_p(FAKE), n, ds["out"]
    if case == "null_inputs":
        host = None
    elif case == "short_buffer":
        nbytes = n - 1
    elif case == "out_shape":
        out = desc((1, 64, 4, 7))
    outp = None if case == "null_out" else ctypes.byref(out)
    ws = lib.ipa_attn_workspace_size(ctypes.byref(p))
    sz = lib.ipa_attn_host_staging_size(ctypes.byref(p))
    st = lib.ipa_attn_fwd_host_packed(ctypes.byref(p), host, ctypes.c_size_t(nbytes), outp, ctypes.c_void_p(FAKE),
                                      ctypes.c_size_t(sz), ctypes.c_void_p(FAKE), ctypes.c_size_t(ws), None,
                                      ctypes.c_void_p(FAKE))
    assert st == expect
