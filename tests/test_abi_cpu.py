"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, sizes workspaces, and rejects bad arguments on the host before
touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

import attention_free_long_b200 as av

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "avey.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"AVEY_API\s+[\w\s\*]*?\b(avey_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("avey_rank", "avey_compress", "avey_dynamic_mix", "avey_layer_forward",
              "avey_rank_workspace_bytes", "avey_layer_workspace_bytes", "avey_device_status",
              "avey_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = av.lib()
    out = subprocess.run(["nm", "-D", "--defined-only", av.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (avey_\w+)", out))
    for n in _declared():
        assert n in exported, n
        assert hasattr(L, n)


def test_header_compiles_as_c():
    src = "#include \"avey.h\"\nint main(void){ return (int)AVEY_OK; }\n"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        "-x", "c", "-", "-o", "/dev/null"], input=src, text=True,
                       capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings():
    L = av.lib()
    for code, name in av.STATUS.items():
        assert L.avey_status_string(code).decode() == name


def test_workspace_sizes():
    # bf16: 1/||x|| per padded row (rows rounded up to 256) + scores fp32
    n, R = 64, 64 * 64
    expect = (8 * R * 4 + 255) // 256 * 256 + (8 * n * n * 4 + 255) // 256 * 256
    assert av.rank_workspace_bytes(av.AVEY_BF16, 8, 4096, 768, 64) == expect
    # fp32: a normalised copy X_hat + scores
    expect32 = (8 * R * 768 * 4 + 255) // 256 * 256 + (8 * n * n * 4 + 255) // 256 * 256
    assert av.rank_workspace_bytes(av.AVEY_F32, 8, 4096, 768, 64) == expect32
    assert av.rank_workspace_bytes(av.AVEY_BF16, 0, 4096, 768, 64) == 0
    T, d, m = 4096, 768, 1536
    b = av.layer_workspace_bytes(av.AVEY_BF16, T, d, m, False)
    assert b == T * m * 4 + T * d * 4
    assert av.layer_workspace_bytes(av.AVEY_BF16, T, d, m, True) == b + T * 4
    assert av.layer_workspace_bytes(av.AVEY_F32, T, d, m, False) == T * m * 4


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below is rejected first


def _rank(**kw):
    a = dict(x=FAKE, dt=av.AVEY_BF16, B=1, N=256, d=64, S=64, k=3, idx=FAKE, w=FAKE, scores=None,
             ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    return av.lib().avey_rank(a["x"], a["dt"], a["B"], a["N"], a["d"], a["S"], a["k"], a["idx"],
                              a["w"], a["scores"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(x=None), 1), (dict(idx=None), 1), (dict(ws=None), 1),
    (dict(B=0), 1), (dict(N=0), 1), (dict(k=0), 1), (dict(d=60), 1),
    (dict(k=33), 2), (dict(S=48), 2), (dict(dt=av.AVEY_BF16X2), 2),
    (dict(ws_bytes=16), 1), (dict(x=ctypes.c_void_p(0x10004)), 1),
    (dict(ws=ctypes.c_void_p(0x10010)), 1),
])
def test_rank_rejects_bad_arguments_on_the_host(kw, code):
    assert _rank(**kw) == code
    assert av.lib().avey_last_error_detail().decode() != ""


def test_compress_rejects_bad_arguments():
    L = av.lib()
    assert L.avey_compress(None, av.AVEY_BF16, 1, 256, 64, 64, 3, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert L.avey_compress(FAKE, av.AVEY_BF16, 1, 256, 64, 48, 3, FAKE, FAKE, FAKE, FAKE, None, None) == 2
    assert L.avey_compress(FAKE, av.AVEY_F32, 1, 256, 64, 128, 3, FAKE, FAKE, FAKE, FAKE, None, None) == 2
    assert L.avey_compress(FAKE, av.AVEY_BF16, 1, 256, 64, 64, 40, FAKE, FAKE, FAKE, FAKE, None, None) == 2


def test_dynamic_mix_rejects_partial_overlap_and_bad_shapes():
    L = av.lib()
    base = 0x100000
    # out starts inside zt but is not the same view
    assert L.avey_dynamic_mix(ctypes.c_void_p(base), 64, av.AVEY_BF16X2, 4, 64, 64, 1e-8,
                              ctypes.c_void_p(base + 128), 64, None) == 1
    assert L.avey_dynamic_mix(FAKE, 64, av.AVEY_BF16, 4, 64, 64, 1e-8, FAKE, 64, None) == 2
    assert L.avey_dynamic_mix(FAKE, 60, av.AVEY_BF16X2, 4, 64, 60, 1e-8, FAKE, 60, None) == 1
    assert L.avey_dynamic_mix(FAKE, 64, av.AVEY_BF16X2, 4, 48, 64, 1e-8, FAKE, 64, None) == 2
    assert L.avey_dynamic_mix(FAKE, 64, av.AVEY_F32, 4, 16, 64, -1.0, FAKE, 64, None) == 1


def test_layer_forward_rejects_bad_arguments():
    L = av.lib()
    p = av.LayerParams(av.AVEY_STATIC, 768, 1536, 768, 64, 1e-8, 0, 0x10000, 0x10000, None, 0x10000)
    args = lambda T=4096, ws=FAKE, wsb=1 << 34: (ctypes.byref(p), av.AVEY_BF16, T, FAKE, None, FAKE,
                                                 None, ws, wsb, None)
    assert L.avey_layer_forward(*args()) == 1  # static layer without V
    p.V = 0x10000
    assert L.avey_layer_forward(*args(T=4000)) == 1  # T not a multiple of S
    assert L.avey_layer_forward(*args(wsb=1024)) == 1  # workspace too small
    p.m_h = 1536
    assert L.avey_layer_forward(*args()) == 1  # m_h must be < m
    p.m_h, p.S = 768, 96
    assert L.avey_layer_forward(*args(T=96 * 42)) == 2  # unsupported split size
    assert L.avey_layer_forward(None, av.AVEY_BF16, 4096, FAKE, None, FAKE, None, FAKE, 1, None) == 1


def test_fp32_activations_may_be_omitted_only_beside_the_bf16_pair():
    # x_in / x_out (and compression's out) may be NULL only on the bf16 path
    # and only when the split pair stands in for them
    L = av.lib()
    p = av.LayerParams(av.AVEY_STATIC, 768, 1536, 768, 64, 1e-8, 0, 0x10000, 0x10000, 0x10000, 0x10000)
    call = lambda dt, xi, xil, xo, xol: L.avey_layer_forward(ctypes.byref(p), dt, 4096, xi, xil, xo, xol,
                                                            FAKE, 1 << 34, None)
    assert call(av.AVEY_BF16, None, None, FAKE, None) == 1   # no residual at all
    assert call(av.AVEY_BF16, FAKE, None, None, None) == 1   # no output at all
    assert call(av.AVEY_F32, None, FAKE, FAKE, None) == 1    # fp32 path needs x_in
    assert call(av.AVEY_F32, FAKE, None, None, FAKE) == 1    # fp32 path needs x_out
    assert "x_in may be NULL" in (call(av.AVEY_BF16, None, None, FAKE, None) and
                                  L.avey_last_error_detail().decode())
    cmp = lambda dt, out, lowp: L.avey_compress(FAKE, dt, 1, 256, 64, 64, 3, FAKE, FAKE, FAKE, out, lowp, None)
    assert cmp(av.AVEY_BF16, None, None) == 1
    assert cmp(av.AVEY_F32, None, FAKE) == 1


def test_kernel_trace_rejects_bad_arguments_and_idles_cleanly():
    L = av.lib()
    assert L.avey_trace_end() == -1                    # no trace active
    assert L.avey_trace_begin(0, None) == 1            # AVEY_ERR_INVALID_ARG: capacity
    assert L.avey_trace_begin(4097, None) == 1
    assert L.avey_trace_end() == -1                    # nothing was started
    assert L.avey_trace_kernel_name(0) is None
    ms = ctypes.c_float()
    assert L.avey_trace_kernel_ms(0, ctypes.byref(ms)) == 1
    assert L.avey_trace_kernel_ms(0, None) == 1


def test_rank_static_reports_the_shape_error_before_the_scratch_limit():
    L = av.lib()
    f = L.avey_rank_static
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    fake = ctypes.c_void_p(256)  # never dereferenced: rejected on the host
    # S = 48 is unsupported, and this shape would also exceed the scratch array
    rc = f(fake, av.AVEY_BF16, 1, 48 * 4096, 64, 48, 3, fake, fake, None)
    assert rc == 2
    assert "S=48" in L.avey_last_error_detail().decode()
    # a valid shape beyond the array is rejected for its size
    rc = f(fake, av.AVEY_BF16, 1, 64 * 4096, 64, 64, 3, fake, fake, None)
    assert rc == 2
    assert "scratch" in L.avey_last_error_detail().decode()
