"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point ``include/svdq.h`` declares, sizes and status strings are
right, and invalid arguments are rejected before anything is launched."""
import ctypes
import os
import re

import pytest

from bit_w4a4_quantized_svdq_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "svdq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_debug_library_exports_and_reports_itself():
    """The debug build (store bounds checks in the kernels, pointer checks on the
    host) exports the same entry points; each build says which it is; the
    extent hook is refused by the release build and checks its arguments in the
    debug build (host-side only here)."""
    from bit_w4a4_quantized_svdq_b200.build import DEBUG_LIB_PATH, LIB_PATH
    rel = ctypes.CDLL(LIB_PATH)
    dbg = ctypes.CDLL(DEBUG_LIB_PATH)
    for name in _declared_functions():
        assert hasattr(dbg, name), name
    for lib in (rel, dbg):
        lib.svdq_debug_limit_extent.argtypes = [ctypes.c_int, ctypes.c_int64]
    assert rel.svdq_debug_build() == 0 and dbg.svdq_debug_build() == 1
    assert rel.svdq_debug_limit_extent(4, 0) == _lib.SVDQ_ERR_UNSUPPORTED
    assert dbg.svdq_debug_limit_extent(0, 10) == _lib.SVDQ_ERR_INVALID_ARG
    assert dbg.svdq_debug_limit_extent(17, 10) == _lib.SVDQ_ERR_INVALID_ARG
    assert dbg.svdq_debug_limit_extent(4, -1) == _lib.SVDQ_ERR_INVALID_ARG
    assert dbg.svdq_debug_limit_extent(16, 0) == _lib.SVDQ_OK
    dbg.svdq_status_string.restype = ctypes.c_char_p
    assert dbg.svdq_status_string(_lib.SVDQ_ERR_BOUNDS).startswith(b"a device store fell outside")


def test_version_and_status_strings():
    lib = _lib.load()
    assert lib.svdq_version() == 100
    assert lib.svdq_status_string(0) == b"ok"
    assert lib.svdq_status_string(3) == b"misaligned pointer or stride"
    assert lib.svdq_status_string(99) == b"unknown status"


def test_sf_bytes():
    lib = _lib.load()
    assert lib.svdq_sf_bytes(1, 64) == 128 * 4
    assert lib.svdq_sf_bytes(128, 512) == 128 * 32
    assert lib.svdq_sf_bytes(129, 512) == 256 * 32
    assert lib.svdq_sf_bytes(4096, 5120) == 4096 * 320
    assert lib.svdq_sf_bytes(10, 48) == 0          # K not a multiple of 64


def test_score_workspace_bytes():
    lib = _lib.load()
    segs, n = _lib.seg_array([(0, 29), (29, 4068), (4068, 4096)])
    b = lib.svdq_score_workspace_bytes(segs, n, 5120)
    assert b > 0 and b % 256 == 0
    assert lib.svdq_score_workspace_bytes(None, 0, 5120) == 0


FAKE = 0x10000  # an aligned non-null "device" pointer; never dereferenced on these paths


def test_calib_rejects_bad_arguments():
    lib = _lib.load()
    z = ctypes.c_void_p
    ok_ptr = z(FAKE)
    # null X
    assert lib.svdq_calib_lambda(None, 8, 64, 64, None, 0, None, 0, 0, ok_ptr, None, ok_ptr, None, ok_ptr,
                                 None) == _lib.SVDQ_ERR_INVALID_ARG
    # K not a multiple of 8
    assert lib.svdq_calib_lambda(ok_ptr, 8, 60, 60, None, 0, None, 0, 0, ok_ptr, None, ok_ptr, None, ok_ptr,
                                 None) == _lib.SVDQ_ERR_INVALID_ARG
    # misaligned X
    assert lib.svdq_calib_lambda(z(FAKE + 2), 8, 64, 64, None, 0, None, 0, 0, ok_ptr, None, ok_ptr, None,
                                 ok_ptr, None) == _lib.SVDQ_ERR_MISALIGNED
    # segment out of range
    segs, n = _lib.seg_array([(0, 9)])
    assert lib.svdq_calib_lambda(ok_ptr, 8, 64, 64, segs, n, None, 0, 0, ok_ptr, None, ok_ptr, None, ok_ptr,
                                 None) == _lib.SVDQ_ERR_INVALID_ARG


def test_quantize_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    # K not a multiple of 64
    assert lib.svdq_quantize_act(p, 4, 96, 96, None, p, None, 0, p, p, None, None,
                                 None) == _lib.SVDQ_ERR_UNSUPPORTED
    # unsupported rank
    assert lib.svdq_quantize_act(p, 4, 128, 128, None, p, p, 8, p, p, p, None,
                                 None) == _lib.SVDQ_ERR_UNSUPPORTED
    # rank without D
    assert lib.svdq_quantize_act(p, 4, 128, 128, None, p, p, 16, p, p, None, None,
                                 None) == _lib.SVDQ_ERR_INVALID_ARG
    # null s_g
    assert lib.svdq_quantize_act(p, 4, 128, 128, None, None, None, 0, p, p, None, None,
                                 None) == _lib.SVDQ_ERR_INVALID_ARG
    # misaligned codes
    assert lib.svdq_quantize_act(p, 4, 128, 128, None, p, None, 0, ctypes.c_void_p(FAKE + 4), p, None, None,
                                 None) == _lib.SVDQ_ERR_MISALIGNED


def test_linear_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    args = dict(a=p, asf=p, sga=p, d=None, r=0, w=p, wsf=p, sgw=p, up=None, bias=None, y=p, ldy=512, dt=0,
                m=128, n=512, k=512)

    def call(**kw):
        a = dict(args, **kw)
        return lib.svdq_linear(a["a"], a["asf"], a["sga"], a["d"], a["r"], a["w"], a["wsf"], a["sgw"], a["up"],
                               a["bias"], a["y"], a["ldy"], a["dt"], a["m"], a["n"], a["k"], None)

    assert call(k=288) == _lib.SVDQ_ERR_UNSUPPORTED          # K % 64
    assert call(n=320, ldy=320) == _lib.SVDQ_ERR_UNSUPPORTED  # N % 128
    # K % 64 and N % 128 pass validation; with no GPU the call stops at the device check
    assert call(k=320, n=384, ldy=384) == _lib.SVDQ_ERR_NO_DEVICE
    assert call(r=16) == _lib.SVDQ_ERR_INVALID_ARG           # rank without D / up
    assert call(r=24, d=p, up=p) == _lib.SVDQ_ERR_UNSUPPORTED
    assert call(dt=2) == _lib.SVDQ_ERR_INVALID_ARG
    assert call(ldy=100) == _lib.SVDQ_ERR_INVALID_ARG         # ldy < N
    assert call(y=ctypes.c_void_p(FAKE + 8)) == _lib.SVDQ_ERR_MISALIGNED
    assert call(sga=None) == _lib.SVDQ_ERR_INVALID_ARG


def test_score_and_residual_reject_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    segs, n = _lib.seg_array([(0, 4)])
    assert lib.svdq_score_lambda(p, p, 4, 64, 64, None, 0, p, p, p, p, 4096, None) == _lib.SVDQ_ERR_INVALID_ARG
    bad, nb = _lib.seg_array([(2, 1)])
    assert lib.svdq_score_lambda(p, p, 4, 64, 64, bad, nb, p, p, p, p, 4096, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_score_lambda(p, p, 4, 64, 64, segs, n, p, p, p, None, 0, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_residual(p, 16, 64, 64, None, None, None, 33, p, None) == _lib.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_residual(p, 16, 64, 64, None, None, None, 4, p, None) == _lib.SVDQ_ERR_INVALID_ARG


def test_device_error_requires_output_pointer():
    lib = _lib.load()
    assert lib.svdq_device_error(None, None) == _lib.SVDQ_ERR_INVALID_ARG


def test_bits_lost_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    assert lib.svdq_bits_lost(None, 64, 1, None, 64, 1, 64, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_bits_lost(p, 64, 1, None, 64, 1, 40, p, None) == _lib.SVDQ_ERR_INVALID_ARG    # K % 16
    assert lib.svdq_bits_lost(p, 32, 1, None, 64, 1, 64, p, None) == _lib.SVDQ_ERR_INVALID_ARG    # ld < K
    assert lib.svdq_bits_lost(p, 64, 1, None, 64, 2, 64, p, None) == _lib.SVDQ_ERR_INVALID_ARG    # no lambda, 2 candidates
    assert lib.svdq_bits_lost(p, 64, 0, p, 64, 1, 64, p, None) == _lib.SVDQ_ERR_INVALID_ARG       # no modality
    assert lib.svdq_bits_lost(p, 64, 1, p, 64, 1, 64, ctypes.c_void_p(FAKE + 4), None) == _lib.SVDQ_ERR_MISALIGNED


def test_lambda_grid_rejects_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    assert lib.svdq_lambda_grid(None, p, 64, p, 3, p, p, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lambda_grid(p, p, 0, p, 3, p, p, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lambda_grid(p, p, 64, p, 0, p, p, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_lambda_grid(p, p, 64, p, 3, p, ctypes.c_void_p(FAKE + 2), p, None) == _lib.SVDQ_ERR_MISALIGNED


def test_mxfp8_sizes_and_bad_arguments():
    lib = _lib.load()
    p = ctypes.c_void_p(FAKE)
    assert lib.svdq_mxfp8_sf_bytes(1, 128) == 128 * 4
    assert lib.svdq_mxfp8_sf_bytes(129, 5120) == 256 * 160
    assert lib.svdq_mxfp8_sf_bytes(4, 96) == 0
    assert lib.svdq_quantize_mxfp8(None, 4, 128, 128, p, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_mxfp8(p, 4, 192, 192, p, p, None) == _lib.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_quantize_mxfp8(p, 4, 128, 100, p, p, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_linear_mxfp8(p, p, p, p, None, None, 256, 4, 256, 128, None) == _lib.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_linear_mxfp8(p, p, p, p, None, p, 256, 4, 256, 192, None) == _lib.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_linear_mxfp8(p, p, p, p, None, p, 256, 4, 200, 128, None) == _lib.SVDQ_ERR_UNSUPPORTED


def test_missing_library_fails_loudly():
    # the CUDA library is the only implementation: without it every call raises
    # instead of falling back to anything else (fresh interpreter: the handle is cached)
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, '.');"
            "from bit_w4a4_quantized_svdq_b200 import _lib\n"
            "try:\n    _lib.load('/nonexistent/libsvdq.so')\nexcept ImportError as e:\n"
            "    print('raised', 'build it' in str(e))\nelse:\n    print('loaded')")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=300)
    assert res.stdout.strip() == "raised True", res.stdout + res.stderr


def test_wrappers_reject_tensors_on_different_devices():
    """The binding makes the tensors' device current for the call, so tensors
    split over two devices (or off the GPU) are refused before any launch."""
    import torch

    from bit_w4a4_quantized_svdq_b200 import ops

    cpu = torch.zeros((4, 8), dtype=torch.uint8)
    meta = torch.empty((4, 8), dtype=torch.uint8, device="meta")
    f32 = torch.zeros(1, dtype=torch.float32)
    with pytest.raises(ValueError, match="different devices"):
        ops.svdq_linear(cpu, cpu, f32, None, meta, cpu, f32, None, None)
    with pytest.raises(ValueError, match="different devices"):
        ops.svdq_score_lambda(cpu.view(torch.int16), meta.view(torch.int16), [(0, 4)])
    with pytest.raises(ValueError, match="CUDA tensors"):
        ops.svdq_quantize_act(cpu.view(torch.int16), None, f32)
    with pytest.raises(ValueError, match="CUDA tensors"):
        ops.svdq_calib_lambda(cpu.view(torch.int16), None, None)


def test_binding_refuses_wrong_types_and_short_buffers():
    """Arguments the kernels read through a bare pointer are checked for dtype,
    dense layout and size before any launch (the checks need no device)."""
    import torch

    from bit_w4a4_quantized_svdq_b200 import ops

    m, n, k, r = 4, 256, 128, 16
    sfa, sfw = ops.sf_bytes(m, k), ops.sf_bytes(n, k)
    good = dict(a_codes=torch.zeros((m, k // 2), dtype=torch.uint8), a_sf=torch.zeros(sfa, dtype=torch.uint8),
                s_g_act=torch.ones(1), d=torch.zeros((m, r)), w_codes=torch.zeros((n, k // 2), dtype=torch.uint8),
                w_sf=torch.zeros(sfw, dtype=torch.uint8), s_g_w=torch.ones(()),
                up=torch.zeros((n, r), dtype=torch.int16), bias=torch.zeros(n, dtype=torch.bfloat16))
    assert ops._check_linear_operands(**good) == (m, n, k, r)
    assert ops._check_linear_operands(**dict(good, d=None, up=None, bias=None)) == (m, n, k, 0)
    bad = [
        (dict(s_g_act=torch.ones(1, dtype=torch.float64)), TypeError),        # wrong dtype
        (dict(a_sf=torch.zeros(sfa - 1, dtype=torch.uint8)), ValueError),     # short scale buffer
        (dict(w_sf=torch.zeros(sfa, dtype=torch.uint8)), ValueError),         # the activation's size, not W's
        (dict(d=torch.zeros((m, r)).t().contiguous().t()), ValueError),       # not contiguous
        (dict(d=torch.zeros((m + 1, r))), ValueError),                        # wrong rows
        (dict(up=torch.zeros((n, r + 16), dtype=torch.int16)), ValueError),   # rank differs from D's
        (dict(up=torch.zeros((n, r), dtype=torch.float16)), TypeError),       # not bf16
        (dict(bias=torch.zeros(n - 1, dtype=torch.int16)), ValueError),       # short bias
        (dict(w_codes=torch.zeros((n, k // 2 + 1), dtype=torch.uint8)), ValueError),  # K differs from A's
        (dict(a_codes=torch.zeros((m, k // 2), dtype=torch.int8)), TypeError),
    ]
    for change, err in bad:
        with pytest.raises(err):
            ops._check_linear_operands(**dict(good, **change))
    # 1/lambda and the tensor scale of the activation quantiser
    ops._check_dense(torch.ones((3, k))[1], (torch.float32,), k, "inv_lambda")   # a row of a candidate grid
    ops._check_dense(torch.ones(()), (torch.float32,), 1, "s_g")                  # a 0-dim scale
    with pytest.raises(ValueError):
        ops._check_dense(torch.ones(k - 1), (torch.float32,), k, "inv_lambda")
    with pytest.raises(ValueError):
        ops._check_dense(None, (torch.float32,), 1, "s_g")
    ops._check_dense(None, (torch.float32,), k, "inv_lambda", optional=True)
    ops._check_matrix(torch.zeros((r, k), dtype=torch.int16), ops._BF16_TYPES, r, k, "down")
    with pytest.raises(ValueError):
        ops._check_matrix(torch.zeros((k, r), dtype=torch.int16).t(), ops._BF16_TYPES, r, k, "down")


def test_header_is_plain_c():
    """include/svdq.h compiles as C99 (and as C++) in a unit that takes the
    address of every entry point it declares, so the boundary needs no C++."""
    import shutil
    import subprocess
    import tempfile
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    names = _declared_functions()
    body = ("#include \"svdq.h\"\ntypedef void (*any_fn)(void);\n" +
            "".join(f"any_fn p_{n} = (any_fn)&{n};\n" for n in names))
    with tempfile.TemporaryDirectory() as d:
        for lang, std, ext in (("c", "-std=c99", "c"), ("c++", "-std=c++17", "cc")):
            src = os.path.join(d, f"unit.{ext}")
            with open(src, "w") as f:
                f.write(body)
            res = subprocess.run([cc, "-x", lang, std, "-Wall", "-Werror", "-pedantic", "-c", src,
                                  "-I", os.path.join(ROOT, "include"), "-o", os.path.join(d, f"unit_{ext}.o")],
                                 capture_output=True, text=True)
            assert res.returncode == 0, res.stderr
