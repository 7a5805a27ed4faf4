"""The C-ABI library builds, loads without a GPU and exports every declared entry point.

Only host-side logic is exercised here (plans, shape validation, workspace
layout, option checks); nothing launches a kernel.
"""
import ctypes
import os
import re

import pytest

from fp8_fp4_moe_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    assert sorted(names) == sorted(binding.EXPORTED)
    for n in names:
        assert hasattr(L, n), n


def test_header_is_plain_c(tmp_path):
    # the boundary is a C ABI: the header compiles as pedantic C99 and C11, not only as C++
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "moe_b200.h"\nint main(void) { moe_plan_t p = 0; (void)p; return 0; }\n')
    for std in ("c99", "c11"):
        r = subprocess.run([gcc, f"-std={std}", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                            os.path.dirname(HEADER), "-c", str(src), "-o", str(tmp_path / f"{std}.o")],
                           capture_output=True, text=True)
        assert r.returncode == 0, r.stderr


def test_a_c_program_links_and_plans_without_a_device(L, tmp_path):
    # a caller in C links the library directly: planning and workspace sizing need no GPU
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.join(ROOT, "fp8_fp4_moe_b200")
    src = tmp_path / "plan.c"
    src.write_text(
        '#include <stdio.h>\n#include "moe_b200.h"\n'
        "int main(void) {\n"
        "  moe_plan_t p = 0;\n"
        "  if (moe_plan(4096, 4096, 14336, 8, 2, 0, &p) != MOE_OK) return 1;\n"
        "  size_t ws = moe_workspace_bytes(p);\n"
        "  moe_plan_destroy(p);\n"
        "  if (moe_plan(4096, 100, 14336, 8, 2, 0, &p) != MOE_ERR_UNSUPPORTED_SHAPE) return 2;\n"
        '  printf("%zu\\n", ws);\n'
        "  return ws > 0 ? 0 : 3;\n"
        "}\n")
    exe = tmp_path / "plan"
    r = subprocess.run([gcc, "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-L", lib_dir, "-lmoe_b200",
                        f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert int(r.stdout) > 0


def test_binding_constants_match_the_header():
    # every MOE_OPT_ / MOE_ERR_ value the binding defines is the header's
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    header = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(MOE_(?:OPT|ERR)_\w+)\s*=\s*(-?\d+)", text)}
    assert len([k for k in header if k.startswith("MOE_OPT_")]) >= 12
    for name, value in header.items():
        assert getattr(binding, name) == value, name


def _plan(L, *shape):
    h = ctypes.c_void_p()
    rc = L.moe_plan(*shape, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("shape", [
    (0, 256, 512, 8, 2, 0),      # T < 1
    (64, 200, 512, 8, 2, 0),     # H % 128
    (64, 256, 500, 8, 2, 0),     # I % 128
    (64, 256, 512, 8, 9, 0),     # k > E
    (64, 256, 512, 8, 0, 0),     # k < 1
    (64, 256, 512, 32, 17, 0),   # k > 16
    (64, 256, 512, 1025, 2, 0),  # E > 1024
    (64, 256, 512, 1024, 2, 1),  # E + shared > 1024
    (64, 256, 512, 8, 2, 2),     # shared not 0/1
])
def test_plan_rejects_unsupported_shapes(L, shape):
    rc, h = _plan(L, *shape)
    assert rc == binding.MOE_ERR_UNSUPPORTED_SHAPE and not h.value


def test_workspace_layout_is_aligned_and_disjoint(L):
    rc, h = _plan(L, 4096, 4096, 14336, 8, 2, 0)
    assert rc == 0
    total = L.moe_workspace_bytes(h)
    T, H, I, k = 4096, 4096, 14336, 2
    rows = T * k
    spans = []
    for name, r in binding.REGIONS.items():
        off, n = ctypes.c_size_t(), ctypes.c_size_t()
        assert L.moe_workspace_region(h, r, ctypes.byref(off), ctypes.byref(n)) == 0
        assert off.value % 256 == 0 and off.value + n.value <= total
        spans.append((off.value, off.value + n.value, name))
    spans.sort()
    for a, b in zip(spans, spans[1:]):
        assert a[1] <= b[0], (a, b)
    sizes = {name: e - s for s, e, name in spans}
    assert sizes["xq"] == rows * H and sizes["hq"] == rows * I and sizes["y"] == rows * H * 2
    off, n = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.moe_workspace_region(h, 99, ctypes.byref(off), ctypes.byref(n)) == binding.MOE_ERR_INVALID_ARG
    L.moe_plan_destroy(h)


def test_options_and_unbound_plan(L):
    rc, h = _plan(L, 64, 256, 512, 8, 2, 0)
    assert rc == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_MAX_SMS, 16) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TIMEOUT_NS, 0) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, binding.MOE_OPT_INJECT_FAULT, 2) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, 12345, 1) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 32, 64):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_SWAP_ROWS, v) == 0
    for v in (-1, 16, 65, 128):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_SWAP_ROWS, v) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 1, 2):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_PAIR_TILES, v) == 0
    for v in (-1, 3):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_PAIR_TILES, v) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 1):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_FUSED, v) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_FUSED, 2) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 1, 2):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_DEPENDENT_LAUNCH, v) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_DEPENDENT_LAUNCH, 3) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 1):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_CHAIN, v) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_CHAIN, 2) == binding.MOE_ERR_INVALID_ARG
    for v in (0, 256):
        assert L.moe_plan_set_option(h, binding.MOE_OPT_L2_TILE_ROWS, v) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_L2_TILE_ROWS, 128) == binding.MOE_ERR_INVALID_ARG
    # H = 256 is not a multiple of 224
    assert L.moe_plan_set_option(h, binding.MOE_OPT_L2_TILE_ROWS, 224) == binding.MOE_ERR_UNSUPPORTED_SHAPE
    rc, h2 = _plan(L, 64, 896, 512, 8, 2, 0)
    assert rc == 0 and L.moe_plan_set_option(h2, binding.MOE_OPT_L2_TILE_ROWS, 224) == 0
    L.moe_plan_destroy(h2)
    # no workspace bound yet: every compute entry point refuses before touching a device
    null = [None] * 9
    assert L.moe_forward(h, *null) == binding.MOE_ERR_WORKSPACE
    assert L.moe_debug_routing(h, *null[:6]) == binding.MOE_ERR_WORKSPACE
    assert L.moe_set_workspace(h, None, 0) == binding.MOE_ERR_WORKSPACE
    assert L.moe_update_bias(h, None, 0.01, None) == binding.MOE_ERR_WORKSPACE
    assert L.moe_update_bias(None, None, 0.01, None) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_forward(None, *null) == binding.MOE_ERR_INVALID_ARG
    L.moe_plan_destroy(h)
    L.moe_plan_destroy(None)


def test_tile_rows_option_and_get_option(L):
    import ctypes as C

    def get(h, key):
        v = C.c_longlong()
        assert L.moe_plan_get_option(h, key, C.byref(v)) == 0
        return v.value

    # few tokens on decode-sized experts (T <= 32, T*k <= 32*E): 32-row tiles by default; more
    # tokens: 128-row tiles, zero-padded while the experts still average <= 32 rows
    rc, h1 = _plan(L, 16, 7168, 2048, 256, 8, 1)
    assert rc == 0 and get(h1, binding.MOE_OPT_TILE_ROWS) == 32 and get(h1, binding.MOE_OPT_ZERO_PAD) == 2
    L.moe_plan_destroy(h1)
    rc, h2 = _plan(L, 8192, 7168, 2048, 256, 8, 1)
    assert rc == 0 and get(h2, binding.MOE_OPT_TILE_ROWS) == 128 and get(h2, binding.MOE_OPT_ZERO_PAD) == 2
    assert L.moe_plan_set_option(h2, binding.MOE_OPT_ZERO_PAD, 1) == 0 and get(h2, binding.MOE_OPT_ZERO_PAD) == 1
    assert L.moe_plan_set_option(h2, binding.MOE_OPT_ZERO_PAD, 3) == binding.MOE_ERR_INVALID_ARG
    L.moe_plan_destroy(h2)
    rc, h = _plan(L, 512, 7168, 2048, 256, 8, 1)
    assert rc == 0 and get(h, binding.MOE_OPT_TILE_ROWS) == 128 and get(h, binding.MOE_OPT_ZERO_PAD) == 1
    assert L.moe_plan_set_option(h, binding.MOE_OPT_ZERO_PAD, 2) == 0 and get(h, binding.MOE_OPT_ZERO_PAD) == 2
    # forced heights; transposed tiles and forced CTA pairs need 128-row tiles
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 128) == 0 and get(h, binding.MOE_OPT_TILE_ROWS) == 128
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 64) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 32) == 0 and get(h, binding.MOE_OPT_TILE_ROWS) == 32
    assert get(h, binding.MOE_OPT_ZERO_PAD) == 2                     # no padding on 32-row tiles
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 0) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_SWAP_ROWS, 64) == 0
    assert get(h, binding.MOE_OPT_TILE_ROWS) == 128                 # transposed tiles need 128 rows
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 32) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, binding.MOE_OPT_SWAP_ROWS, 0) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_TILE_ROWS, 32) == 0
    assert L.moe_plan_set_option(h, binding.MOE_OPT_SWAP_ROWS, 32) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, binding.MOE_OPT_PAIR_TILES, 2) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_set_option(h, binding.MOE_OPT_PAIR_TILES, 1) == 0
    # other keys report what was set; the linear2 tile height resolves (H = 7168 = 32 * 224)
    assert get(h, binding.MOE_OPT_PAIR_TILES) == 1
    assert get(h, binding.MOE_OPT_DEPENDENT_LAUNCH) == 0          # automatic: off above 64 tokens
    assert get(h, binding.MOE_OPT_L2_TILE_ROWS) == 256
    assert L.moe_plan_set_option(h, binding.MOE_OPT_L2_TILE_ROWS, 224) == 0 and get(h, binding.MOE_OPT_L2_TILE_ROWS) == 224
    v = C.c_longlong()
    assert L.moe_plan_get_option(h, 12345, C.byref(v)) == binding.MOE_ERR_INVALID_ARG
    assert L.moe_plan_get_option(None, binding.MOE_OPT_GRAPH, C.byref(v)) == binding.MOE_ERR_INVALID_ARG
    L.moe_plan_destroy(h)


def test_dense_gemm_validation_without_a_device(L):
    assert L.moe_gemm_workspace_bytes(0, 128, 128) == 0
    assert L.moe_gemm_workspace_bytes(4, 100, 128) == 0          # N % 128
    assert L.moe_gemm_workspace_bytes(4, 128, 96) == 0           # K % 128
    n = L.moe_gemm_workspace_bytes(300, 256, 512)
    # status + bookkeeping + the 3-entry row-tile table, 3 row tiles x 4 K-blocks of 512-byte
    # atoms, 1 n-tile x 4 of 1 KB units
    assert n == 6 * 256 + 3 * 4 * 512 + 4 * 1024
    null = [None] * 6
    assert L.moe_gemm_fp8_fp4(4, 100, 128, *null, 0, None) == binding.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_gemm_fp8_fp4(4, 128, 128, *null, 0, None) == binding.MOE_ERR_INVALID_ARG


def test_error_strings(L):
    for code in range(-6, 1):
        assert L.moe_error_string(code)
    assert L.moe_error_string(-99) == b"unknown error"


def test_route_noalloc_binding_rejects_mismatched_shapes_before_the_library():
    """The binding validates every shape (and the device) before any pointer reaches the C ABI."""
    import torch

    from fp8_fp4_moe_b200 import binding
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    W = torch.zeros(8, 256, dtype=torch.float32)
    b = torch.zeros(8, dtype=torch.float32)
    with pytest.raises(ValueError):
        binding.route_noalloc(x[0], W, b, 2)                       # x not [T, H]
    with pytest.raises(ValueError):
        binding.route_noalloc(x, W[:, :128], b, 2)                 # W_router too narrow
    with pytest.raises(ValueError):
        binding.route_noalloc(x, W, b[:7], 2)                      # bias of the wrong length
    with pytest.raises(ValueError):
        binding.route_noalloc(x, W, b, 2)                          # CPU tensors
