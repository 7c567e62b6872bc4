"""Host-only checks of the C ABI (include/m2rnn.h): the library loads, exports
every declared entry point, sizes workspaces and rejects bad arguments before
touching the device.  No kernel is launched here."""
import ctypes
import re
import os

import pytest

from non_linear_matrix_persistent_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_exports_match_header(L):
    header = open(os.path.join(ROOT, "include", "m2rnn.h")).read()
    declared = set(re.findall(r"\b(m2rnn_[a-z_]+)\s*\(", header))
    assert declared == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def _dims(B=2, H=3, T=5, K=64, V=64, mode=0, C=16, G=0, logit=0):
    return _lib.Dims(B, H, T, K, V, mode, C, G, logit)


def test_workspace_size(L):
    # 128 (b, h) pairs fill the GPU: one CTA per pair, the forward needs only the status word
    assert L.m2rnn_workspace_size(_dims(B=8, H=16), 0) == 256
    # 6 pairs of 64 x 64 states (384 rows <= 148 x 8): the row kernel, 8 rows
    # per CTA, so 8 slices per pair whose partial readouts the workspace keeps
    assert L.m2rnn_workspace_size(_dims(), 0) == 256 + 8 * (2 * 3 * 5 * 64) * 4
    # 16 pairs of 64 x 64 (1024 rows): still the row kernel; 32 pairs (2048 rows): the
    # tensor-core kernel with 4 slices of 16 rows
    assert L.m2rnn_workspace_size(_dims(B=1, H=16), 0) == 256 + 8 * (16 * 5 * 64) * 4
    assert L.m2rnn_workspace_size(_dims(B=2, H=16), 0) == 256 + 4 * (32 * 5 * 64) * 4
    # other widths take the tensor-core kernel: 6 pairs split the 64 rows into 4 slices
    assert L.m2rnn_workspace_size(_dims(V=32), 0) == 256 + 4 * (2 * 3 * 5 * 32) * 4
    assert L.m2rnn_workspace_size(_dims(mode=1), 0) == 256   # fp32 debug mode: no slices
    assert L.m2rnn_workspace_size(_dims(mode=1), 1) > 256
    assert L.m2rnn_workspace_size(_dims(K=48), 0) == 0
    assert L.m2rnn_workspace_size(_dims(mode=7), 0) == 0
    assert L.m2rnn_workspace_size(None, 0) == 0


def test_status_strings(L):
    for s in range(7):
        assert _lib.status_string(s).startswith("M2RNN_")
    assert _lib.status_string(99) == "M2RNN_ERR_UNKNOWN"


def _fwd(L, d, ptrs=None, ws_bytes=1 << 20):
    p = dict(k=4096, v=4096, q=4096, f=4096, W=4096, H0=None, y=4096, HT=None, ckpt=None, ws=4096)
    p.update(ptrs or {})
    return L.m2rnn_forward(d, p["k"], p["v"], p["q"], p["f"], p["W"], p["H0"], p["y"], p["HT"], p["ckpt"],
                           p["ws"], ws_bytes, None)


def test_forward_argument_errors(L):
    # every case fails validation, so nothing reaches the device
    assert _fwd(L, None) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(K=24)) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _fwd(L, _dims(V=256)) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _fwd(L, _dims(C=0)) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _fwd(L, _dims(B=-1)) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(mode=4)) == _lib.ERR_INVALID_ARG
    # the register-resident forward covers V = 64, K <= 64 only (checked before any launch)
    assert _fwd(L, _dims(K=128, mode=_lib.MODE_BF16_MMA_SYNC)) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _fwd(L, _dims(V=32, mode=_lib.MODE_BF16_MMA_SYNC)) == _lib.ERR_UNSUPPORTED_SHAPE
    assert _fwd(L, _dims(), {"k": None}) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(), {"y": None}) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(), {"ws": None}) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(), {"q": 4100}) == _lib.ERR_MISALIGNED
    assert _fwd(L, _dims(), {"HT": 4104}) == _lib.ERR_MISALIGNED
    assert _fwd(L, _dims(), ws_bytes=100) == _lib.ERR_WORKSPACE
    # zero-sized batch: nothing to do
    assert _fwd(L, _dims(B=0)) == _lib.OK


def test_backward_argument_errors(L):
    def bwd(d, **kw):
        p = dict(k=4096, v=4096, q=4096, f=4096, W=4096, ckpt=4096, dy=4096, dHT=None, dk=4096, dv=4096,
                 dq=4096, df=4096, dW=4096, dH0=4096, ws=4096, ws_bytes=1 << 40)
        p.update(kw)
        return L.m2rnn_backward(d, p["k"], p["v"], p["q"], p["f"], p["W"], p["ckpt"], p["dy"], p["dHT"], p["dk"],
                                p["dv"], p["dq"], p["df"], p["dW"], p["dH0"], p["ws"], p["ws_bytes"], None)
    assert bwd(_dims(), ckpt=None) == _lib.ERR_INVALID_ARG
    assert bwd(_dims(), dW=None) == _lib.ERR_INVALID_ARG
    assert bwd(_dims(), dy=4097) == _lib.ERR_MISALIGNED
    assert bwd(_dims(mode=1), ws_bytes=256) == _lib.ERR_WORKSPACE
    assert bwd(_dims(K=8)) == _lib.ERR_UNSUPPORTED_SHAPE
    # the fast-tanh and register-resident modes are forward only
    assert bwd(_dims(mode=_lib.MODE_BF16_TC_FAST_TANH)) == _lib.ERR_INVALID_ARG
    assert bwd(_dims(mode=_lib.MODE_BF16_MMA_SYNC)) == _lib.ERR_INVALID_ARG


def test_tc_backward_every_shape_has_a_workspace(L):
    """The tensor-core backward takes every K, V in {16, 32, 64, 128} with a
    checkpoint stride of at most 16.  V = 64 with K >= 32 and a stride within
    the extended-operand kernel's tensor-memory scratch (8 steps for K >= 64,
    16 for K = 32) needs only the dW partials (one per 64-row slice); longer
    strides there, and the other shapes, take the general-shape kernel, whose
    workspace adds 2·C·KS·MX scratch values per CTA, except at V = 128 with a
    stride its tensor memory holds (8 steps for 32-row slices, 16 for 16-row
    ones); K = 128 at V = 128 runs four 32-row slices per pair, whose dv and
    df partials (4·B·H·T·(V + 1) fp32) are summed after the kernel."""
    B, H, T, C = 2, 3, 5, 4
    for K in (16, 32, 64, 128):
        for V in (16, 32, 64, 128):
            assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=K, V=V, C=C), 1) > 256, (K, V)
            # a longer stride gets only the status word, and the call is rejected before any launch
            assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=K, V=V, C=17), 1) == 256, (K, V)
            st = L.m2rnn_backward(_dims(B=B, H=H, T=T, K=K, V=V, C=17), *([4096] * 7), None, *([4096] * 7),
                                  1 << 40, None)
            assert st == _lib.ERR_UNSUPPORTED_SHAPE, (K, V)
    def pad(n):
        return 256 + (n + 255) // 256 * 256
    for K, cmax, nsl in ((32, 16, 1), (64, 8, 1), (128, 8, 2)):
        for C in (1, 4, cmax):
            assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=K, V=64, C=C), 1) == pad(
                4 * B * H * nsl * 64 * 64), (K, C)
    # K = V = 64 beyond 8 steps: the general-shape kernel (one 64-row slice, MX = 64)
    assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=64, V=64, C=12), 1) == pad(
        4 * (B * H * 64 * 64 + 2 * 12 * B * H * 64 * 64))
    ncta = B * H * 4
    # V = 128 keeps a chunk of at most 8 steps (32-row slices) on chip: no scratch then
    assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=128, V=128, C=C), 1) == pad(
        4 * (ncta * 128 * 128 + 4 * B * H * T * 129))
    assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=128, V=128, C=12), 1) == pad(
        4 * (ncta * 128 * 128 + 2 * 12 * ncta * 32 * 128 + 4 * B * H * T * 129))
    # 16-row slices (K = 16) hold 16 steps
    assert L.m2rnn_workspace_size(_dims(B=B, H=H, T=T, K=16, V=128, C=16), 1) == pad(4 * B * H * 128 * 128)


def test_fast_tanh_mode_workspace(L):
    fast = _lib.MODE_BF16_TC_FAST_TANH
    for B, H in ((2, 3), (8, 16)):
        assert L.m2rnn_workspace_size(_dims(B=B, H=H, mode=fast), 0) == L.m2rnn_workspace_size(_dims(B=B, H=H), 0)
    assert L.m2rnn_workspace_size(_dims(mode=fast), 1) == 0
    assert L.m2rnn_workspace_size(_dims(mode=4), 0) == 0


def test_mma_sync_mode_workspace(L):
    mma = _lib.MODE_BF16_MMA_SYNC
    assert L.m2rnn_workspace_size(_dims(mode=mma), 0) == 256   # one CTA per pair, no slices
    assert L.m2rnn_workspace_size(_dims(mode=mma), 1) == 0     # forward only


def test_grouped_qk_heads(L):
    """k / q head groups: 0 or H = one per head; otherwise a proper divisor of
    H.  The backward keeps per-head dk and dq (2·B·H·T·K fp32) before summing
    each group; the forward needs nothing extra."""
    for mode in (0, 1):
        for B, H in ((2, 4), (8, 16)):
            plain = [L.m2rnn_workspace_size(_dims(B=B, H=H, mode=mode), bw) for bw in (0, 1)]
            assert [L.m2rnn_workspace_size(_dims(B=B, H=H, mode=mode, G=H), bw) for bw in (0, 1)] == plain
            for G in (1, 2):
                d = _dims(B=B, H=H, mode=mode, G=G)
                assert L.m2rnn_workspace_size(d, 0) == plain[0]
                assert L.m2rnn_workspace_size(d, 1) == plain[1] + 2 * B * H * 5 * 64 * 4
    for G in (-1, 2, 4):   # negative, not a divisor of H = 3, more groups than heads
        assert L.m2rnn_workspace_size(_dims(G=G), 0) == 0
        assert _fwd(L, _dims(G=G)) == _lib.ERR_INVALID_ARG
    assert _fwd(L, _dims(B=0, H=0, G=1)) == _lib.ERR_INVALID_ARG


def test_api_grouped_shapes_are_checked_on_the_host():
    import torch
    from non_linear_matrix_persistent_b200 import api
    B, H, T, K, V = 1, 4, 2, 16, 16
    bf = dict(dtype=torch.bfloat16)
    v = torch.zeros(B, H, T, V, **bf)
    assert api.dims_of(torch.zeros(B, 2, T, K, **bf), v).qk_heads == 2
    assert api.dims_of(torch.zeros(B, 4, T, K, **bf), v).qk_heads == 0   # one per head
    with pytest.raises(ValueError):
        api.dims_of(torch.zeros(B, 3, T, K, **bf), v)


def test_gate_logit_flag(L):
    for mode in (0, 1):
        for bw in (0, 1):
            assert L.m2rnn_workspace_size(_dims(mode=mode, logit=1), bw) == L.m2rnn_workspace_size(_dims(mode=mode), bw)
    for bad in (-1, 2):
        assert L.m2rnn_workspace_size(_dims(logit=bad), 0) == 0
        assert _fwd(L, _dims(logit=bad)) == _lib.ERR_INVALID_ARG


def test_status_query_rejects_null(L):
    assert L.m2rnn_get_device_status(None, None) == _lib.ERR_INVALID_ARG


def test_dims_struct_matches_header():
    """The ctypes m2rnn_dims has the header's int fields in the header's order
    (a missing or reordered field would shift every later one)."""
    header = open(os.path.join(ROOT, "include", "m2rnn.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    body = re.search(r"typedef struct \{(.*?)\} m2rnn_dims;", header, flags=re.S).group(1)
    names = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            assert decl.startswith("int "), decl
            names += [n.strip() for n in decl[4:].split(",")]
    assert names == [n for n, _ in _lib.Dims._fields_]
    assert all(t is ctypes.c_int for _, t in _lib.Dims._fields_)


def test_binding_signatures_match_header(L):
    """Each ctypes declaration has exactly the parameter count of the header prototype
    (a missing parameter shifts every later argument, e.g. the stream handle)."""
    header = open(os.path.join(ROOT, "include", "m2rnn.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    for name in _lib.EXPORTS:
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", header)
        assert m, name
        params = [x for x in m.group(1).split(",") if x.strip() and x.strip() != "void"]
        assert len(getattr(L, name).argtypes) == len(params), (name, len(params))


def test_api_mode_flags_are_checked_before_any_launch():
    import torch
    from non_linear_matrix_persistent_b200 import api
    B, H, T, K, V = 1, 1, 2, 16, 16
    f32 = dict(dtype=torch.float32)
    k, q = torch.zeros(B, H, T, K, **f32), torch.zeros(B, H, T, K, **f32)
    v, f, W = torch.zeros(B, H, T, V, **f32), torch.zeros(B, H, T, **f32), torch.zeros(H, V, V, **f32)
    with pytest.raises(TypeError):          # the alternatives need bf16 inputs
        api.forward(k, v, q, f, W, fast_tanh=True)
    with pytest.raises(TypeError):
        api.forward(k, v, q, f, W, mma_sync=True)
    bf = [t.to(torch.bfloat16) for t in (k, v, q)]
    with pytest.raises(ValueError):         # one alternative at a time
        api.forward(bf[0], bf[1], bf[2], f, W.to(torch.bfloat16), fast_tanh=True, mma_sync=True)
    with pytest.raises(ValueError):         # step needs the state buffer
        api.step(k[:, :, 0], v[:, :, 0], q[:, :, 0], f[:, :, 0], W, None)


def test_header_is_plain_c(tmp_path):
    """include/m2rnn.h compiles as strict C99 (a C caller needs no C++ or CUDA headers)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text('#include "m2rnn.h"\n'
                   "size_t ws(void) { m2rnn_dims d = {1, 1, 1, 16, 16, M2RNN_MODE_FP32_DEBUG, 16, 0, 0};\n"
                   "  return m2rnn_workspace_size(&d, 0); }\n")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                        os.path.join(ROOT, "include"), "-c", str(src), "-o", str(tmp_path / "use.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_api_rejects_bad_tensors_before_any_launch():
    """Shape, dtype and device problems are reported by the binding before it
    allocates a workspace or calls the library (CPU tensors stand in for any
    tensor that is not on the expected CUDA device)."""
    import torch
    from non_linear_matrix_persistent_b200 import api
    B, H, T, K, V = 1, 2, 3, 16, 16
    bf = dict(dtype=torch.bfloat16)
    k, q = torch.zeros(B, H, T, K, **bf), torch.zeros(B, H, T, K, **bf)
    v, W = torch.zeros(B, H, T, V, **bf), torch.zeros(H, V, V, **bf)
    f = torch.zeros(B, H, T)
    with pytest.raises(ValueError, match="CUDA"):
        api.forward(k, v, q, f, W)
    with pytest.raises(TypeError):                  # integer inputs select no mode
        api.forward(k.to(torch.int32), v, q, f, W)
    with pytest.raises(ValueError):                 # k with a head count that does not divide H
        api.dims_of(torch.zeros(B, 3, T, K, **bf), v)
    d = api.dims_of(k, v, ckpt_stride=4, f_is_logit=True)
    assert (d.B, d.H, d.T, d.K, d.V, d.ckpt_stride, d.qk_heads, d.f_is_logit) == (B, H, T, K, V, 4, 0, 1)
    assert d.mode == 0 and api.dims_of(k.float(), v.float()).mode == 1


def test_enum_values_match_header():
    """Status codes and modes of the binding carry the header's values."""
    header = open(os.path.join(ROOT, "include", "m2rnn.h")).read()
    header = re.sub(r"/\*.*?\*/", "", header, flags=re.S)
    vals = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(M2RNN_[A-Z0-9_]+)\s*=\s*(\d+)", header)}
    py = {"M2RNN_OK": _lib.OK, "M2RNN_ERR_INVALID_ARG": _lib.ERR_INVALID_ARG,
          "M2RNN_ERR_UNSUPPORTED_SHAPE": _lib.ERR_UNSUPPORTED_SHAPE, "M2RNN_ERR_MISALIGNED": _lib.ERR_MISALIGNED,
          "M2RNN_ERR_WORKSPACE": _lib.ERR_WORKSPACE, "M2RNN_ERR_CUDA": _lib.ERR_CUDA,
          "M2RNN_ERR_DEVICE_TIMEOUT": _lib.ERR_DEVICE_TIMEOUT,
          "M2RNN_MODE_BF16_TC": _lib.MODE_BF16_TC, "M2RNN_MODE_FP32_DEBUG": _lib.MODE_FP32_DEBUG,
          "M2RNN_MODE_BF16_TC_FAST_TANH": _lib.MODE_BF16_TC_FAST_TANH,
          "M2RNN_MODE_BF16_MMA_SYNC": _lib.MODE_BF16_MMA_SYNC}
    assert vals == py
