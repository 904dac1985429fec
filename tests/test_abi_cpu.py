"""The C ABI library on a machine without a GPU: it builds, loads, exports every
symbol that include/sqa.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

import sparse_query_attention_sqa_b200 as sqa
from sparse_query_attention_sqa_b200 import build as sqa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sqa_build.build()
    return sqa.load_library()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(sqa_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"sqa_fwd", "sqa_bwd", "sqa_bwd_workspace_bytes", "sqa_last_error"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} is declared but not exported"


def test_library_is_in_tree_and_built_for_sm100a():
    assert os.path.dirname(sqa.library_path()) == os.path.join(ROOT, "sparse_query_attention_sqa_b200")
    with open(os.path.join(ROOT, "sparse_query_attention_sqa_b200", "build.py")) as f:
        assert "arch=compute_100a,code=sm_100a" in f.read()


def test_status_strings(lib):
    assert lib.sqa_status_string(0) == b"ok"
    assert lib.sqa_status_string(1) == b"invalid argument"
    assert lib.sqa_version() >= 100


def _fwd(lib, ptrs, shape, scale=0.0):
    return lib.sqa_fwd(*ptrs, sqa.Shape(*shape), 1, ctypes.c_float(scale), None)


GOOD = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000]


@pytest.mark.parametrize("shape,code", [
    ((1, 8, 6, 4, 16), 1),     # H_q not a multiple of H_kv
    ((0, 8, 8, 4, 16), 1),     # empty batch
    ((1, 0, 8, 4, 16), 1),     # empty sequence
    ((1, 8, 8, 0, 16), 1),     # no KV heads
    ((1, 8, 8, 4, 48), 2),     # unsupported head dim
    ((1, 8, 8, 4, 8), 2),      # unsupported head dim
    ((1, 8, 256, 1, 16), 2),   # group larger than 128
])
def test_fwd_rejects_bad_shapes_before_launch(lib, shape, code):
    assert _fwd(lib, GOOD, shape) == code
    assert lib.sqa_last_error() != b""


def test_fwd_rejects_null_and_misaligned_pointers(lib):
    for i in range(5):
        ptrs = list(GOOD)
        ptrs[i] = 0
        assert _fwd(lib, ptrs, (1, 8, 8, 4, 16)) == 1
    ptrs = list(GOOD)
    ptrs[0] += 8  # q not 16-byte aligned
    assert _fwd(lib, ptrs, (1, 8, 8, 4, 16)) == 2
    assert _fwd(lib, GOOD, (1, 8, 8, 4, 16), scale=float("nan")) == 1


def test_bwd_rejects_bad_arguments_before_launch(lib):
    s = sqa.Shape(1, 64, 8, 4, 16)
    need = lib.sqa_bwd_workspace_bytes(s)
    assert need > 0
    p = [0x10000 * (i + 1) for i in range(10)]
    # workspace too small
    assert lib.sqa_bwd(*p, need - 1, s, 1, ctypes.c_float(0.0), None) == 1
    # null pointer
    q = list(p)
    q[3] = 0
    assert lib.sqa_bwd(*q, need, s, 1, ctypes.c_float(0.0), None) == 1
    # misaligned workspace
    q = list(p)
    q[9] += 16
    assert lib.sqa_bwd(*q, need, s, 1, ctypes.c_float(0.0), None) == 2
    # bad shape
    assert lib.sqa_bwd(*p, need, sqa.Shape(1, 64, 6, 4, 16), 1, ctypes.c_float(0.0), None) == 1
    assert lib.sqa_bwd_workspace_bytes(sqa.Shape(1, 64, 6, 4, 16)) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sqa, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sqa, "_lib", None)
    with pytest.raises(ImportError):
        sqa.load_library()


def test_exp2_selftest_rejects_null_pointers_before_launch(lib):
    f = lib.sqa_selftest_exp2_poly
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(None, None, 0, None) == 0  # nothing to do
    assert f(None, 0x100, 4, None) == 1
    assert f(0x100, 0x104, 4, None) == 1  # y misaligned


def test_decode_rejects_bad_arguments_before_launch(lib):
    f = lib.sqa_decode
    vp = ctypes.c_void_p
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, sqa.Shape, ctypes.c_float, vp]
    f.restype = ctypes.c_int
    s = sqa.Shape(2, 300, 8, 4, 16)
    need = lib.sqa_decode_workspace_bytes(s)
    assert need > 0
    ok = [0x1000, 0x2000, 0x3000, 0, 0x4000, 0x5000, 0x6000]
    assert f(*ok[:3], None, *ok[4:], need, sqa.Shape(2, 300, 6, 4, 16), 0.0, None) == 1  # H_q % H_kv
    assert f(*ok[:3], None, *ok[4:], need, sqa.Shape(2, 300, 8, 4, 48), 0.0, None) == 2  # head dim
    assert f(None, *ok[1:3], None, *ok[4:], need, s, 0.0, None) == 1  # null q
    assert f(ok[0], 0x2008, ok[2], None, *ok[4:], need, s, 0.0, None) == 2  # cache not 16-byte aligned
    assert f(*ok[:3], None, *ok[4:], need - 1, s, 0.0, None) == 1  # workspace too small
    assert lib.sqa_decode_workspace_bytes(sqa.Shape(0, 300, 8, 4, 16)) == 0


def _decode_ws_expected(B, N, Hq, Hkv, dh):
    """Workspace rule of sqa_decode: one (o, m, l) record of dh + 2 floats per
    (sequence, K/V head, range, query head of the group), for the most ranges
    either split path can take: the shared-memory path's fixed ranges (4 chunks
    of 256/128/64 positions at dh <= 32/64/128) or the register-resident path's
    shortest range (16 steps of 2048/dh cache rows, i.e. 16 * 2048 / dh / H_kv
    positions) when the group has at most 4 heads and H_kv is a power of two
    no larger than 2048/dh."""
    g = Hq // Hkv
    span = 4 * (256 if dh <= 32 else (128 if dh == 64 else 64))
    n = -(-N // span)
    step = 2048 // dh
    if 1 <= g <= 4 and Hkv & (Hkv - 1) == 0 and Hkv <= step:
        n = max(n, -(-N // (16 * step // Hkv)))
    return -(-(B * Hkv * n * g * (dh + 2) * 4) // 256) * 256


@pytest.mark.parametrize("shape", [(32, 32768, 8, 4, 16), (8, 65536, 8, 4, 128), (2, 3000, 128, 1, 16),
                                   (2, 500, 6, 3, 32), (2, 300, 16, 16, 128), (2, 300, 32, 32, 128), (1, 1, 4, 1, 64)])
def test_decode_workspace_covers_both_split_paths(lib, shape):
    assert lib.sqa_decode_workspace_bytes(sqa.Shape(*shape)) == _decode_ws_expected(*shape)


def test_plain_c_client_builds_links_and_runs(lib, tmp_path):
    """include/sqa.h compiles as C11 (warnings as errors), a C program links
    against libsqa.so, and its calls give the documented results without a GPU."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    pkg = os.path.join(ROOT, "sparse_query_attention_sqa_b200")
    exe = str(tmp_path / "c_client")
    subprocess.run([gcc, "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "abi", "c_client.c"), "-L", pkg, "-lsqa", f"-Wl,-rpath,{pkg}",
                    "-o", exe], check=True, capture_output=True, text=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(got["version"]) == lib.sqa_version()
    assert int(got["bwd_workspace"]) == lib.sqa_bwd_workspace_bytes(sqa.Shape(32, 1024, 8, 4, 16))
    assert int(got["decode_workspace"]) == lib.sqa_decode_workspace_bytes(sqa.Shape(32, 32768, 8, 4, 16))
    assert int(got["decode_workspace_invalid"]) == 0
    invalid, unsupported = "1", "2"
    assert got["fwd_null"] == invalid and got["fwd_group"] == invalid
    assert got["fwd_dh"] == unsupported and got["fwd_misaligned"] == unsupported
    assert got["bwd_small_workspace"] == invalid and got["decode_null"] == invalid
    assert got["timing_bad_kernel"] == invalid
    assert got["status_string_ok"] == "1" and got["last_error_nonempty"] == "1"


def _bwd_ws_expected(B, N, Hq, Hkv, dh):
    """Workspace rule of sqa_bwd: -lse*log2(e) and -D per stacked-tile slot
    (B * H_kv * n_qtiles * 128 fp32 each); for dh <= 32 also the fp32 dQ
    accumulator [B][N][H_q][dh] (at dh 64 and 128 dQ comes from its own kernel
    with no accumulator); every part rounded up to 256 bytes."""
    def a256(x):
        return -(-x // 256) * 256

    g = Hq // Hkv
    T = 128 // g
    slots = B * Hkv * -(-N // T) * 128
    total = 2 * a256(slots * 4)
    if dh <= 32:
        total += a256(B * N * Hq * dh * 4)
    return total


@pytest.mark.parametrize("shape", [(32, 1024, 8, 4, 16), (2, 65536, 8, 4, 128), (1, 1000, 6, 2, 32),
                                   (3, 77, 128, 1, 64), (1, 1, 16, 16, 16), (1, 200000, 8, 4, 16)])
def test_bwd_workspace_follows_its_layout(lib, shape):
    assert lib.sqa_bwd_workspace_bytes(sqa.Shape(*shape)) == _bwd_ws_expected(*shape)


def test_layer_rejects_bad_arguments_before_launch(lib):
    s = sqa.LayerShape(2, 256, 256, 8, 4, 16)
    need_f = lib.sqa_layer_workspace_bytes(s, 0)
    need_b = lib.sqa_layer_workspace_bytes(s, 1)
    # forward: the rotary table [N][dh/2] of (cos, sin); backward adds dO, dQ,
    # dK, dV and the core's workspace
    assert need_f == 256 * 8 * 8
    core = lib.sqa_bwd_workspace_bytes(sqa.Shape(2, 256, 8, 4, 16))
    assert need_b == need_f + 2 * (2 * 256 * 128 * 2) + 2 * (2 * 256 * 64 * 2) + core
    assert lib.sqa_layer_workspace_bytes(sqa.LayerShape(2, 256, 250, 8, 4, 16), 0) == 0  # d % 8 != 0
    p = 0x10000
    args = [p] * 9 + [p, need_f]
    st = lib.sqa_layer_fwd(*([0] + args[1:]), s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG
    st = lib.sqa_layer_fwd(*args[:10], need_f - 1, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"workspace" in lib.sqa_last_error()
    st = lib.sqa_layer_fwd(*args, s, 1, 0.0, -1.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"rope_base" in lib.sqa_last_error()
    st = lib.sqa_layer_fwd(*args, sqa.LayerShape(2, 256, 250, 8, 4, 16), 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_UNSUPPORTED
    st = lib.sqa_layer_fwd(*args, sqa.LayerShape(2, 256, 256, 6, 4, 16), 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG
    bargs = [p] * 13 + [need_b]
    st = lib.sqa_layer_bwd(*bargs[:12], 0, need_b, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG
    st = lib.sqa_layer_bwd(*bargs[:13], need_b - 256, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"workspace" in lib.sqa_last_error()


def test_block_rejects_bad_arguments_before_launch(lib):
    b = sqa._block_lib()
    s = sqa.BlockShape(2, 256, 256, 8, 4, 16, 768)
    need = b.sqa_block_state_bytes(s)
    assert need > 0
    assert b.sqa_block_state_bytes(sqa.BlockShape(2, 256, 256, 8, 4, 16, 700)) == 0  # hidden % 8 != 0
    assert b.sqa_block_state_bytes(sqa.BlockShape(2, 256, 16384, 8, 4, 16, 768)) == 0  # d > 8192
    p = 0x10000
    w = sqa.BlockWeights(*([p] * 7))
    st = b.sqa_block_fwd(p, ctypes.byref(w), p, p, need - 1, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"state" in b.sqa_last_error()
    w0 = sqa.BlockWeights(*([p] * 6 + [0]))
    st = b.sqa_block_fwd(p, ctypes.byref(w0), p, p, need, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"weight" in b.sqa_last_error()
    g = sqa.BlockGrads(*([p] * 7))
    st = b.sqa_block_bwd(p, p, ctypes.byref(w), p, need, p, ctypes.byref(g), s, 1, 0.0, -2.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG and b"rope_base" in b.sqa_last_error()
    st = b.sqa_block_bwd(p, p, ctypes.byref(w), p, need, p, None, s, 1, 0.0, 10000.0, None)
    assert st == sqa.SQA_ERR_INVALID_ARG


def test_exp2_rate_probe_rejects_bad_arguments_before_launch(lib):
    f = lib.sqa_selftest_exp2_rate
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    assert f(None, 1, 1, None) == 1
    assert f(0x100, 0, 1, None) == 1
    assert f(0x100, 65536, 1, None) == 1
    assert f(0x100, 1, 0, None) == 1
    assert f(0x100, 1, (1 << 20) + 1, None) == 1


def _fwd_ws_expected(B, N, Hq, Hkv, dh, causal, sms=148):
    """Workspace rule of sqa_fwd_with_workspace: nothing unless the problem is
    small (dh <= 64, pairs of Q tiles and single Q tiles both under half the
    SMs) and ranges of `chunk` key tiles (the smallest even count, at least 2,
    whose items do not outnumber the SMs) shorten the longest Q tile's walk
    by at least 6 key tiles per slot; then fp32 partial outputs
    [B*H_kv][n_qtiles][ranges of the longest tile][128][dh], their
    log-sum-exps [..][128] and int counters [B*H_kv][n_qtiles][128], each
    rounded up to 256 bytes."""
    def a256(x):
        return -(-x // 256) * 256

    g = Hq // Hkv
    T = 128 // g
    n_qt = -(-N // T)
    n_bh = B * Hkv
    NK = 128 if dh == 128 else 64
    if dh > 64 or -(-n_qt // 2) * n_bh >= sms // 2 or n_qt * n_bh >= sms // 2:
        return 0
    nkv = [-(-(min(N, (qt + 1) * T) if causal else N) // NK) for qt in range(n_qt)]
    chunk = 2
    while chunk < nkv[-1] and n_bh * sum(-(-n // chunk) for n in nkv) > sms:
        chunk += 2
    if -(-nkv[-1] // 2) - chunk // 2 < 6:
        return 0
    slots = n_bh * n_qt * -(-nkv[-1] // chunk) * 128
    return a256(slots * dh * 4) + a256(slots * 4) + a256(n_bh * n_qt * 128 * 4)


@pytest.mark.parametrize("shape", [(1, 1024, 8, 4, 16), (1, 333, 12, 4, 16), (1, 390, 8, 4, 64), (1, 2000, 2, 1, 32),
                                   (32, 1024, 8, 4, 16), (2, 65536, 8, 4, 128), (1, 300, 8, 4, 128), (1, 64, 8, 4, 16),
                                   (1, 200, 16, 1, 64), (1, 4096, 2, 1, 16), (1, 2500, 3, 1, 64), (1, 513, 6, 1, 16),
                                   (1, 1500, 6, 1, 16), (1, 1000, 2, 2, 16)])
@pytest.mark.parametrize("causal", [0, 1])
def test_fwd_workspace_follows_its_rule(lib, shape, causal):
    assert lib.sqa_fwd_workspace_bytes(sqa.Shape(*shape), causal) == _fwd_ws_expected(*shape, causal)


def test_fwd_workspace_sizes_of_two_small_shapes(lib):
    """B=1, N=4096, 2/1 heads, dh 16, causal: 64 Q tiles, ranges of 18 key
    tiles (16 would make 160 items for 148 SMs), at most 4 per Q tile:
    64 * 4 * 128 slots of 16 + 1 floats, 8192 counters.  The SQAT-m
    layer-sized forward (B=1, N=1024, 8/4) would save 5 key tiles per slot
    (8 -> 3): none."""
    assert lib.sqa_fwd_workspace_bytes(sqa.Shape(1, 4096, 2, 1, 16), 1) == 32768 * 17 * 4 + 8192 * 4
    assert lib.sqa_fwd_workspace_bytes(sqa.Shape(1, 1024, 8, 4, 16), 1) == 0


def test_fwd_with_workspace_rejects_bad_arguments_before_launch(lib):
    f = lib.sqa_fwd_with_workspace
    s = sqa.Shape(1, 4096, 2, 1, 16)
    need = lib.sqa_fwd_workspace_bytes(s, 1)
    assert need > 0
    ptrs = [0x1000, 0x2000, 0x3000, 0x4000, 0x5000]
    assert f(*ptrs, None, need, s, 1, 0.0, None) == 1  # workspace needed
    assert f(*ptrs, 0x6010, need, s, 1, 0.0, None) == 2  # workspace not 256-byte aligned
    assert f(*ptrs, 0x6000, need - 1, s, 1, 0.0, None) == 1  # workspace too small
    assert f(None, *ptrs[1:], 0x6000, need, s, 1, 0.0, None) == 1  # null q
    assert f(*ptrs, 0x6000, need, sqa.Shape(1, 4096, 3, 2, 16), 1, 0.0, None) == 1  # H_q % H_kv
