"""The C-ABI library on the host: it loads without a GPU, exports every symbol
the header declares, and rejects bad arguments with status codes before it
touches the device.  No compute call runs here."""
import ctypes
import os
import re

import pytest

import rmsnorm_linear_projection_flashnorm_b200 as fnb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flashnorm.h")


@pytest.fixture(scope="module")
def L():
    fnb.build()
    return fnb.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fn_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fn_fold_weights", "fn_norm_proj", "fn_norm_proj_swiglu", "fn_workspace_size",
                     "fn_query_device_status", "fn_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert fnb.fn_version() == 1


def test_status_strings(L):
    for code in range(9):
        assert fnb.status_string(code).startswith("FN_")


# fake, never-dereferenced device addresses: validation must reject before use
A = 1 << 20          # 16-byte aligned
B = 1 << 30
C = 1 << 34
WS = 1 << 36


def np_(x=A, M=4, d=256, Wp=B, scales=None, wt=0, N=512, eps=1e-6, y=C, ws=WS, ws_bytes=1 << 30, swiglu=False):
    f = fnb.fn_norm_proj_swiglu if swiglu else fnb.fn_norm_proj
    return f(x, M, d, Wp, scales, wt, N, eps, y, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(M=-1), fnb.FN_ERR_INVALID_ARG),
    (dict(d=0), fnb.FN_ERR_INVALID_ARG),
    (dict(N=0), fnb.FN_ERR_INVALID_ARG),
    (dict(eps=-1e-6), fnb.FN_ERR_INVALID_ARG),
    (dict(eps=float("nan")), fnb.FN_ERR_INVALID_ARG),
    (dict(eps=float("inf")), fnb.FN_ERR_INVALID_ARG),
    (dict(wt=7), fnb.FN_ERR_INVALID_ARG),
    (dict(d=100), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(N=500), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(wt=1, d=192, scales=A + (1 << 18)), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(M=1 << 31), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(x=None), fnb.FN_ERR_INVALID_ARG),
    (dict(Wp=None), fnb.FN_ERR_INVALID_ARG),
    (dict(y=None), fnb.FN_ERR_INVALID_ARG),
    (dict(ws=None), fnb.FN_ERR_WORKSPACE),
    (dict(wt=1, scales=None), fnb.FN_ERR_INVALID_ARG),
    (dict(x=A + 8), fnb.FN_ERR_ALIGNMENT),
    (dict(y=C + 2), fnb.FN_ERR_ALIGNMENT),
    (dict(Wp=B + 4), fnb.FN_ERR_ALIGNMENT),
    (dict(ws=WS + 8), fnb.FN_ERR_ALIGNMENT),
    (dict(y=A + 16), fnb.FN_ERR_ALIAS),          # y overlaps x
    (dict(y=B + 1024), fnb.FN_ERR_ALIAS),        # y overlaps W'
    (dict(ws=C + 256), fnb.FN_ERR_ALIAS),        # workspace overlaps y
    (dict(swiglu=True, y=B + 307200), fnb.FN_ERR_ALIAS),  # W' is [d, 2N]: 512 KB
])
def test_norm_proj_rejects_bad_arguments(L, kw, code):
    assert np_(**kw) == code


def test_empty_batch_is_a_noop(L):
    assert np_(M=0, x=None, y=None, ws=None) == fnb.FN_OK
    assert np_(M=0, swiglu=True, x=None, y=None, ws=None) == fnb.FN_OK


GS = (1 << 37) + 4096     # global scale: 4-byte aligned
Q = 1 << 38
SF = 1 << 39


def nvfp4_(x=A, M=4, d=256, Wp=B, scales=None, wt=0, N=512, eps=1e-6, gs=GS, q=Q, sf=SF, ws=WS,
           ws_bytes=1 << 30):
    return fnb.fn_norm_proj_swiglu_nvfp4(x, M, d, Wp, scales, wt, N, eps, gs, q, sf, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(M=-1), fnb.FN_ERR_INVALID_ARG),
    (dict(gs=None), fnb.FN_ERR_INVALID_ARG),
    (dict(q=None), fnb.FN_ERR_INVALID_ARG),
    (dict(sf=None), fnb.FN_ERR_INVALID_ARG),
    (dict(N=500), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(q=Q + 8), fnb.FN_ERR_ALIGNMENT),
    (dict(sf=SF + 8), fnb.FN_ERR_ALIGNMENT),
    (dict(gs=GS + 2), fnb.FN_ERR_ALIGNMENT),
    (dict(q=A + 16), fnb.FN_ERR_ALIAS),          # codes overlap x
    (dict(sf=B + 64), fnb.FN_ERR_ALIAS),         # scale bytes overlap W'
    (dict(sf=Q + 512), fnb.FN_ERR_ALIAS),        # codes [4, 256] bytes: 1 KB
    (dict(gs=SF + 4), fnb.FN_ERR_ALIAS),         # global scale inside the scale bytes
    (dict(q=WS + 256), fnb.FN_ERR_ALIAS),        # codes inside the workspace
])
def test_nvfp4_rejects_bad_arguments(L, kw, code):
    assert nvfp4_(**kw) == code


def test_nvfp4_empty_batch_is_a_noop(L):
    assert nvfp4_(M=0, x=None, gs=None, q=None, sf=None, ws=None) == fnb.FN_OK


@pytest.mark.parametrize("kw,code", [
    (dict(d=0), fnb.FN_ERR_INVALID_ARG),
    (dict(W0=None), fnb.FN_ERR_INVALID_ARG),
    (dict(g=None), fnb.FN_ERR_INVALID_ARG),
    (dict(out_type=3), fnb.FN_ERR_INVALID_ARG),
    (dict(out_type=1, scales=None), fnb.FN_ERR_INVALID_ARG),
    (dict(N=100), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(out_type=1, d=192), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(W0=A + 2), fnb.FN_ERR_ALIGNMENT),
    (dict(Wp=A + 64), fnb.FN_ERR_ALIAS),
])
def test_fold_rejects_bad_arguments(L, kw, code):
    args = dict(W0=A, W1=None, g=B, d=256, N=512, out_type=0, Wp=C, scales=WS)
    args.update(kw)
    st = fnb.fn_fold_weights(args["W0"], args["W1"], args["g"], args["d"], args["N"], args["out_type"],
                             args["Wp"], args["scales"], None)
    assert st == code


def test_workspace_size_is_monotone_in_m_bucket(L):
    sizes = [fnb.fn_workspace_size(m, 4096, 6144, 0, 0) for m in (1, 16, 17, 32, 33, 64)]
    assert sizes[0] == sizes[1] and sizes[2] == sizes[3] and sizes[4] == sizes[5]
    assert sizes[0] < sizes[2] < sizes[4]
    assert fnb.fn_workspace_size(65, 4096, 6144, 0, 0) == 256
    assert fnb.fn_workspace_size(8, 4096, 14336, 0, 1) > fnb.fn_workspace_size(8, 4096, 14336, 0, 0)


def test_workspace_size_fp8_tile_path(L):
    """fp8 weights above 64 rows: the header, the x_hi and x_lo code planes
    (M d bytes each), and per (row, 128-deep k block) 2^-e and a partial sum
    of squares; from 1024 rows at least the bf16 weight copy that the NVFP4
    and partial outputs use.  The fixed 8 MiB array of the no-allocation entry
    point therefore cannot hold fp8 at 8192 rows of the fp8 workload."""
    fp8 = fnb.FN_W_FP8_E4M3_B128
    r256 = lambda n: (n + 255) // 256 * 256
    M, d, N = 256, 5120, 13824
    assert fnb.fn_workspace_size(M, d, N, fp8, 1) == 256 + 2 * r256(M * d) + 2 * r256((d // 128) * M * 4)
    assert fnb.fn_workspace_size(8192, d, N, fp8, 1) >= 256 + d * 2 * N * 2
    assert fnb.fn_workspace_size(8192, d, N, fp8, 0) > 8 << 20
    assert fnb.fn_workspace_size(65, 1024, 1024, fp8, 0) <= 8 << 20
    # from 33 rows bf16 output takes the promotion kernel, NVFP4 and partial
    # outputs still the decode kernel: the size covers both
    for m in (33, 48, 64):
        need = 256 + 2 * r256(m * d) + 2 * r256((d // 128) * m * 4)
        assert fnb.fn_workspace_size(m, d, N, fp8, 1) >= need
        assert fnb.fn_workspace_size(m, d, N, fp8, 1) >= fnb.fn_workspace_size(32, d, N, fp8, 1)


def test_set_debug_validates_keys(L):
    assert fnb.fn_set_debug(99, 1) == fnb.FN_ERR_INVALID_ARG
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 0) == fnb.FN_ERR_INVALID_ARG
    assert fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 5) == fnb.FN_ERR_INVALID_ARG
    assert fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 4) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_FORCE_PATH, 0) == fnb.FN_OK
    assert fnb.fn_set_debug(fnb.FN_DEBUG_WAIT_BUDGET_NS, 2_000_000_000) == fnb.FN_OK


def test_set_debug_decode_groups_and_pair_tile(L):
    """The cluster decode plan knob: mode 0..2, a forced plan's T (0..3) in bits
    4..7 and S (0..8) in bits 8..11, nothing above; the pair-tile knob 0..2."""
    G, P = fnb.FN_DEBUG_DECODE_GROUPS, fnb.FN_DEBUG_PAIR_TILE
    for v in (0, 1, 2, 2 | (3 << 4) | (4 << 8), 2 | (1 << 4) | (8 << 8)):
        assert fnb.fn_set_debug(G, v) == fnb.FN_OK
    for v in (-1, 3, 2 | (4 << 4), 2 | (3 << 4) | (9 << 8), 1 << 12):
        assert fnb.fn_set_debug(G, v) == fnb.FN_ERR_INVALID_ARG
    assert fnb.fn_set_debug(G, 0) == fnb.FN_OK
    for v in (0, 1, 2):
        assert fnb.fn_set_debug(P, v) == fnb.FN_OK
    for v in (-1, 3):
        assert fnb.fn_set_debug(P, v) == fnb.FN_ERR_INVALID_ARG
    assert fnb.fn_set_debug(P, 0) == fnb.FN_OK


def test_no_device_means_no_launch(L):
    """Valid arguments without a GPU fail cleanly (no device), never crash."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = np_()
    assert st in (fnb.FN_ERR_CUDA, fnb.FN_ERR_UNSUPPORTED_DEVICE)


P = 1 << 40           # partial buffer


def partial_(x=A, M=4, d=256, Wp=B, scales=None, wt=0, ncols=512, part=P, ws=WS, ws_bytes=1 << 30):
    return fnb.fn_norm_proj_partial(x, M, d, Wp, scales, wt, ncols, part, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(M=-1), fnb.FN_ERR_INVALID_ARG),
    (dict(part=None), fnb.FN_ERR_INVALID_ARG),
    (dict(x=None), fnb.FN_ERR_INVALID_ARG),
    (dict(ncols=500), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(d=96), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(wt=1, d=192, scales=A + (1 << 18)), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(part=P + 8), fnb.FN_ERR_ALIGNMENT),
    (dict(part=A + 512), fnb.FN_ERR_ALIAS),      # overlaps x
    (dict(part=WS + 1024), fnb.FN_ERR_ALIAS),    # inside the workspace
    (dict(ws=P + 4096), fnb.FN_ERR_ALIAS),       # partial is (4*512 + 4) floats
])
def test_partial_rejects_bad_arguments(L, kw, code):
    assert partial_(**kw) == code


def post_(part=P, M=4, N=256, swiglu=0, d_total=1024, eps=1e-6, y=C):
    return fnb.fn_post_scale(part, M, N, swiglu, d_total, eps, y, None)


@pytest.mark.parametrize("kw,code", [
    (dict(M=-1), fnb.FN_ERR_INVALID_ARG),
    (dict(d_total=0), fnb.FN_ERR_INVALID_ARG),
    (dict(eps=-1.0), fnb.FN_ERR_INVALID_ARG),
    (dict(N=200), fnb.FN_ERR_UNSUPPORTED_SHAPE),
    (dict(part=None), fnb.FN_ERR_INVALID_ARG),
    (dict(y=None), fnb.FN_ERR_INVALID_ARG),
    (dict(y=C + 4), fnb.FN_ERR_ALIGNMENT),
    (dict(y=P + 1024), fnb.FN_ERR_ALIAS),
    (dict(swiglu=1, y=P + 8192), fnb.FN_ERR_ALIAS),   # SwiGLU partial: 4 x 512 + 4 floats
])
def test_post_scale_rejects_bad_arguments(L, kw, code):
    assert post_(**kw) == code


def test_partial_and_post_scale_empty_batch(L):
    assert partial_(M=0, x=None, part=None, ws=None) == fnb.FN_OK
    assert post_(M=0, part=None, y=None) == fnb.FN_OK


def test_post_scale_rejects_a_grid_too_large(L):
    # (2^31 - 1) rows x 2^21 columns: more than 2^31 blocks of 256 threads
    assert post_(M=(1 << 31) - 1, N=1 << 21) == fnb.FN_ERR_UNSUPPORTED_SHAPE


def test_abi_is_usable_from_plain_c(L, tmp_path):
    """Compile a C11 program against the header with gcc (no C++, no CUDA
    headers), link it to the library, and run it: the declarations are valid
    C, every symbol links, and argument errors come back as status codes."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(fnb.LIB_PATH)
    exe = str(tmp_path / "abi_from_c")
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), src, "-o", exe,
                        "-L", lib_dir, "-lflashnorm", f"-Wl,-rpath,{lib_dir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")   # validation only: no device is touched
    r = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_validation_never_crashes_and_returns_a_status(L):
    """Random argument combinations (sizes, alignments, overlaps, null
    pointers) on a host without a GPU: every call returns one of the declared
    status codes, and with no device none can succeed (M > 0).  Skipped where
    a GPU is visible: random addresses must never reach a launch."""
    import torch
    from hypothesis import given, settings, strategies as st
    if torch.cuda.is_available():
        pytest.skip("random device addresses are only safe without a GPU")

    codes = {fnb.FN_OK, fnb.FN_ERR_INVALID_ARG, fnb.FN_ERR_UNSUPPORTED_SHAPE, fnb.FN_ERR_ALIGNMENT,
             fnb.FN_ERR_ALIAS, fnb.FN_ERR_WORKSPACE, fnb.FN_ERR_CUDA, fnb.FN_ERR_UNSUPPORTED_DEVICE}
    ptr = st.one_of(st.none(), st.integers(1, 1 << 44))
    size = st.integers(-2, 1 << 33)

    @settings(max_examples=300, deadline=None, database=None)
    @given(M=size, d=size, N=size, wt=st.integers(-1, 2), eps=st.floats(allow_nan=True, allow_infinity=True),
           x=ptr, w=ptr, y=ptr, ws=ptr, ws_bytes=st.integers(0, 1 << 34), swiglu=st.booleans(),
           fp4=st.booleans(), part=st.booleans())
    def run(M, d, N, wt, eps, x, w, y, ws, ws_bytes, swiglu, fp4, part):
        if fp4:
            st_ = fnb.fn_norm_proj_swiglu_nvfp4(x, M, d, w, None, wt, N, eps, ws, y, x, ws, ws_bytes, None)
        elif part:
            st_ = fnb.fn_norm_proj_partial(x, M, d, w, None, wt, N, y, ws, ws_bytes, None)
        else:
            f = fnb.fn_norm_proj_swiglu if swiglu else fnb.fn_norm_proj
            st_ = f(x, M, d, w, None, wt, N, eps, y, ws, ws_bytes, None)
        assert st_ in codes
        assert st_ != fnb.FN_OK or M == 0

    run()
