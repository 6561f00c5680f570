"""The C ABI without a GPU: the library loads, exports every function its header declares,
and rejects invalid arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import bit_weight_only_w2_b200 as lb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(lowbit_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return lb.load()


def test_header_declares_entry_points():
    names = declared_functions()
    for required in ("lowbit_pack", "lowbit_unpack", "lowbit_gemm", "lowbit_gemm_batch", "lowbit_gemm_ex",
                     "lowbit_packed_words", "lowbit_device_status", "lowbit_status_string",
                     "lowbit_gemm_workspace_size"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_host_functions(lib):
    assert lib.lowbit_version() >= 100
    assert lib.lowbit_status_string(0) == b"LOWBIT_OK"
    assert lib.lowbit_status_string(5) == b"LOWBIT_ERR_BAD_CODE"
    assert lib.lowbit_status_string(99) == b"LOWBIT_ERR_UNKNOWN"
    assert lib.lowbit_packed_words(9216, 3072, 2) == 9216 * 3072 // 16
    assert lib.lowbit_packed_words(4, 64, 1) == 8
    assert lib.lowbit_packed_words(4, 48, 1) == 0      # K not a multiple of 32
    assert lib.lowbit_packed_words(4, 64, 3) == 0      # bits
    assert lib.lowbit_packed_words(-1, 64, 2) == 0
    assert lib.lowbit_status_string(8) == b"LOWBIT_ERR_WORKSPACE"
    assert lib.lowbit_gemm_workspace_size(4608, 3072) == 4608 * 3072 * 2 + 4608 * 4
    assert lib.lowbit_gemm_workspace_size(1, 64) == 256 + 256
    assert lib.lowbit_gemm_workspace_size(-1, 64) == 0


A = 1 << 20  # a fake 256-byte-aligned address: never dereferenced, checks fail first
WS = 1 << 30  # fake workspace size, large enough for every shape below


@pytest.mark.parametrize("args,expect", [
    (dict(bits=3), 1),
    (dict(group_size=0), 1),
    (dict(K=100), 1),                       # K not a multiple of the group size
    (dict(zeros=A), 1),                     # zeros with bits != 4
    (dict(bits=4), 1),                      # bits 4 without zeros
    (dict(X=0), 1),                         # NULL input
    (dict(X=A + 2), 2),                     # misaligned
    (dict(Y=A + 8), 2),
    (dict(group_size=32, K=256), 3),        # GPU path takes groups of 64 / 128 only
    (dict(N=100), 3),                       # N % 8
    (dict(bits=1, K=192, group_size=64), 3),  # binary needs K % 128
    (dict(M=-1), 1),
    (dict(ws=0), 8),                        # no workspace
    (dict(ws=A + 16), 8),                   # workspace not 256-byte aligned
    (dict(ws_bytes=16 * 256 * 2), 8),       # too small (row factors missing)
])
def test_gemm_rejects_before_launch(lib, args, expect):
    a = dict(M=16, N=128, K=256, bits=2, group_size=128, X=A, Wp=A, scales=A, zeros=0, Y=A, ws=A, ws_bytes=WS)
    a.update(args)
    st = lib.lowbit_gemm(a["M"], a["N"], a["K"], a["bits"], a["group_size"], a["X"], a["Wp"], a["scales"],
                         a["zeros"] or None, a["Y"], a["ws"] or None, a["ws_bytes"], None)
    assert st == expect, lb.STATUS.get(st)


def test_gemm_ex_rejects_bad_tile(lib):
    st = lib.lowbit_gemm_ex(16, 128, 256, 2, 128, A, A, A, None, A, A, WS, 48, 0, 0, None)
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 128, 256, 2, 128, A, A, A, None, A, A, WS, 16, 0, 9, None)
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 128, 256, 2, 128, A, A, A, None, A, A, WS, 16, 20, 0, None)   # rows % 8
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 128, 256, 2, 128, A, A, A, None, A, A, WS, 16, 136, 0, None)  # rows > 128
    assert st == 3
    # 256 rows = a tile per CTA pair: only with 256-token tiles (or the automatic width)
    st = lib.lowbit_gemm_ex(16, 256, 256, 2, 128, A, A, A, None, A, A, WS, 16, 256, 0, None)
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 256, 256, 2, 128, A, A, A, None, A, A, WS, 1, 256, 0, None)
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 512, 256, 2, 128, A, A, A, None, A, A, WS, 0, 264, 0, None)
    assert st == 3
    # the small-M kernel (tile_tokens = 1) serves at most 16 tokens
    st = lib.lowbit_gemm_ex(17, 128, 256, 2, 128, A, A, A, None, A, A, WS, 1, 0, 0, None)
    assert st == 3
    st = lib.lowbit_gemm_ex(16, 128, 256, 2, 128, A, A, A, None, A, A, WS, 1, 12, 0, None)      # rows % 8
    assert st == 3


def test_batch_validates_all_first(lib):
    good = lb.GemmDesc(16, 128, 256, 2, 128, A, A, A, None, A)
    bad = lb.GemmDesc(16, 128, 256, 3, 128, A, A, A, None, A)
    arr = (lb.GemmDesc * 2)(good, bad)
    assert lib.lowbit_gemm_batch(arr, 2, A, WS, None) == 1
    assert lib.lowbit_gemm_batch(arr, 1, A, 1024, None) == 8      # workspace too small for the first
    assert lib.lowbit_gemm_batch(None, -1, A, WS, None) == 1
    assert lib.lowbit_gemm_batch(None, 0, None, 0, None) == 0


def test_empty_problems_are_noops(lib):
    assert lib.lowbit_gemm(0, 128, 256, 2, 128, A, A, A, None, A, None, 0, None) == 0
    assert lib.lowbit_gemm(16, 0, 256, 2, 128, A, A, A, None, A, None, 0, None) == 0
    assert lib.lowbit_pack(None, 0, 64, 2, None, None) == 0


def test_pack_rejects_before_launch(lib):
    assert lib.lowbit_pack(A, 4, 48, 1, A, None) == 1       # K % 32
    assert lib.lowbit_pack(A, 4, 64, 3, A, None) == 1
    assert lib.lowbit_pack(A + 1, 4, 64, 2, A, None) == 2
    assert lib.lowbit_unpack(None, 4, 64, 2, A, None) == 1


def test_binding_workspace_size_matches_library():
    """The Python binding's closed-form workspace size equals lowbit_gemm_workspace_size."""
    import bit_weight_only_w2_b200 as lb
    for M, K in [(1, 64), (16, 2560), (512, 9728), (4608, 12288), (7, 192), (0, 64), (3, 128)]:
        assert lb._workspace_size_fast(M, K) == lb.workspace_size(M, K), (M, K)


def test_status_strings_cover_the_enum(lib):
    for code, name in lb.STATUS.items():
        assert lib.lowbit_status_string(code) == name.encode()


def test_fail_next_validates_its_argument(lib):
    assert lib.lowbit_test_fail_next(-1) == 1
    assert lib.lowbit_test_fail_next(4) == 1
    assert lib.lowbit_test_fail_next(0) == 0      # cancel: nothing pending afterwards


def test_debug_build_exports_the_same_abi():
    """liblowbit_debug.so (device-side index checks) exports every declared entry point and says
    it is the checked build; the release build says it is not and launches no self-test."""
    dbg = lb.load_debug()
    for name in declared_functions():
        assert hasattr(dbg, name), f"{name} missing from the debug build"
    assert dbg.lowbit_debug_checks_enabled() == 1
    rel = lb.load()
    assert rel.lowbit_debug_checks_enabled() == 0
    assert rel.lowbit_selftest_index_check(None) == 3     # LOWBIT_ERR_UNSUPPORTED, before any CUDA call


# ---- the Python binding checks shapes and devices before calling the library (CPU tensors: the
# shape checks come first, so a mismatch is reported before the CUDA-device check)
def _cpu_args(M=16, N=128, K=256, bits=2, g=128):
    import torch
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    packed = torch.zeros((N, K * bits // 32), dtype=torch.int32)
    s = torch.zeros((K // g, N), dtype=torch.float16)
    z = torch.zeros((K // g, N), dtype=torch.float16) if bits == 4 else None
    return x, packed, s, z


@pytest.mark.parametrize("bad,match", [
    ("packed_rows", "packed: expected shape"),
    ("packed_cols", "packed: expected shape"),
    ("scales_transposed", "scales: expected shape"),
    ("zeros_shape", "zeros: expected the scales' shape"),
    ("out_shape", "out: expected shape"),
    ("x_1d", "x: expected a contiguous 2-D"),
    ("packed_dtype", "packed: expected a contiguous"),
    ("x_noncontig", "x: expected a contiguous"),
])
def test_binding_rejects_mismatched_tensors(bad, match):
    import torch
    bits = 4 if bad == "zeros_shape" else 2
    g = 64 if bits == 4 else 128
    x, packed, s, z = _cpu_args(bits=bits, g=g)
    out = None
    if bad == "packed_rows":
        packed = torch.zeros((120, packed.shape[1]), dtype=torch.int32)
    elif bad == "packed_cols":
        packed = torch.zeros((packed.shape[0], packed.shape[1] - 4), dtype=torch.int32)
    elif bad == "scales_transposed":
        s = torch.zeros((128, 256 // g), dtype=torch.float16)
    elif bad == "zeros_shape":
        z = torch.zeros((1, 128), dtype=torch.float16)
    elif bad == "out_shape":
        out = torch.zeros((16, 120), dtype=torch.bfloat16)
    elif bad == "x_1d":
        x = torch.zeros(16 * 256, dtype=torch.bfloat16)
    elif bad == "packed_dtype":
        packed = packed.to(torch.int64)
    elif bad == "x_noncontig":
        x = torch.zeros((256, 16), dtype=torch.bfloat16).t()
    with pytest.raises(ValueError, match=match):
        lb.gemm(x, packed, s, z, bits, g, out=out)


def test_binding_rejects_cpu_tensors_and_bad_descs():
    x, packed, s, z = _cpu_args()
    with pytest.raises(ValueError, match="CUDA tensor"):
        lb.gemm(x, packed, s, z, 2, 128)
    import torch
    y = torch.zeros((16, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        lb.make_desc(x, packed, s, z, y, 2, 128)
    with pytest.raises(ValueError, match="out: expected shape"):
        lb.make_desc(x, packed, s, z, torch.zeros((16, 64), dtype=torch.bfloat16), 2, 128)
    with pytest.raises(ValueError, match="packed: 8 words"):
        lb.unpack(torch.zeros((2, 4), dtype=torch.int32), 4, 64, 2)


def test_binding_without_the_library_raises(tmp_path):
    """A copy of the Python package with no built library refuses to load instead of running
    anything else: the product path has no CPU fallback."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "bit_weight_only_w2_b200")
    dst = tmp_path / "bit_weight_only_w2_b200"
    dst.mkdir()
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            shutil.copy(os.path.join(pkg, f), dst / f)
    code = ("import bit_weight_only_w2_b200 as lb, sys\n"
            "assert lb.__file__.startswith(sys.argv[1]), lb.__file__\n"
            "try:\n"
            "    lb.load()\n"
            "except FileNotFoundError as e:\n"
            "    print('raised', e)\n"
            "else:\n"
            "    raise SystemExit('loaded without a library')\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], cwd=str(tmp_path), capture_output=True,
                       text=True, timeout=300, env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode == 0, r.stderr + r.stdout
    assert "raised" in r.stdout and "liblowbit.so is missing" in r.stdout
