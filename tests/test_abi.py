"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every symbol include/fa.h declares, and rejects bad arguments before any
launch."""

import ctypes
import os
import re

import pytest

import io_aware_exact_forward_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = _header_functions()
    for n in ("fa_forward", "fa_backward", "fa_decode_splitkv", "fa_backward_workspace_bytes",
              "fa_decode_workspace_bytes", "fa_check", "fa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = fa.load_library()
    for n in _header_functions():
        assert hasattr(lib, n), n
        assert n in fa.SIGNATURES, f"binding lacks a signature for {n}"


def test_status_strings():
    lib = fa.load_library()
    for code, name in fa.STATUS.items():
        assert lib.fa_status_string(code).decode() == name


NULL = None


@pytest.mark.parametrize("args,expect", [
    # (B, Hq, Hkv, Tq, Tk, d, scale, causal)
    ((1, 1, 1, 16, 16, 96, 1.0, 0), 2),      # unsupported head dim
    ((1, 3, 2, 16, 16, 64, 1.0, 0), 1),      # Hq % Hkv != 0
    ((1, 1, 1, 16, 16, 64, 1.0, 2), 1),      # causal not 0/1
    ((1, 1, 1, -1, 16, 64, 1.0, 0), 1),      # negative length
    ((1, 1, 1, 16, 16, 64, float("nan"), 0), 1),
    ((1, 1, 1, 16, 16, 64, 1.0, 0), 1),      # null pointers
    ((0, 1, 1, 16, 16, 64, 1.0, 0), 0),      # empty batch: no-op
    ((1, 1, 1, 0, 16, 64, 1.0, 0), 0),       # empty query: no-op
])
def test_forward_rejects_bad_arguments_on_host(args, expect):
    lib = fa.load_library()
    assert lib.fa_forward(NULL, NULL, NULL, NULL, NULL, *args, NULL) == expect


def test_forward_alignment_checked_before_launch():
    lib = fa.load_library()
    buf = (ctypes.c_uint8 * 64)()
    base = ctypes.addressof(buf)
    odd = ctypes.c_void_p(base + (16 - base % 16) + 2)
    st = lib.fa_forward(odd, odd, odd, odd, odd, 1, 1, 1, 16, 16, 64, 1.0, 0, NULL)
    assert st == 3


def test_backward_and_decode_argument_checks():
    lib = fa.load_library()
    assert lib.fa_backward(*([NULL] * 9), NULL, 0, 1, 1, 1, 16, 16, 80, 1.0, 0, NULL) == 2
    assert lib.fa_backward(*([NULL] * 9), NULL, 0, 1, 2, 3, 16, 16, 64, 1.0, 0, NULL) == 1
    # decode: G must be 1,2,4,8; chunk a multiple of 64; chunk*G <= 4096
    assert lib.fa_decode_splitkv(*([NULL] * 6), NULL, 0, 2, 32, 2, 1024, 128, 0.1, 256, NULL) == 2
    assert lib.fa_decode_splitkv(*([NULL] * 6), NULL, 0, 2, 32, 8, 1024, 128, 0.1, 100, NULL) == 1
    assert lib.fa_decode_splitkv(*([NULL] * 6), NULL, 0, 2, 32, 4, 1024, 128, 0.1, 2048, NULL) == 1
    assert lib.fa_decode_splitkv(*([NULL] * 6), NULL, 0, 2, 32, 8, 1024, 128, 0.1, 256, NULL) == 1


def test_workspace_sizes():
    lib = fa.load_library()
    B, Hq, T, d = 2, 4, 100, 64
    ws = lib.fa_backward_workspace_bytes(B, Hq, 2, T, T, d)
    assert ws >= B * T * Hq * d * 4 + B * Hq * T * 4
    assert ws % 256 == 0
    dws = lib.fa_decode_workspace_bytes(64, 32, 32768, 128, 256)
    n = 32768 // 256
    assert dws >= 64 * 32 * n * (128 + 1) * 4
    assert lib.fa_decode_workspace_bytes(1, 1, 10, 96, 256) == 0


def test_product_path_has_no_oracle_dependency():
    """The package must never import or call the CPU oracle."""
    pkg = os.path.join(ROOT, "io_aware_exact_forward_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower() or f.endswith((".cu", ".cuh", ".h")) and "oracle" not in text, f
                assert "import oracle" not in text and "from oracle" not in text, f


def test_window_entry_points_reject_bad_window_on_host():
    lib = fa.load_library()
    # window must be >= 1 (and at most 2^30); checked before any pointer
    for w in (0, -3, (1 << 30) + 1):
        assert lib.fa_forward_window(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 16, 16, 64, 1.0, w, NULL) == 1
        assert lib.fa_backward_window(*([NULL] * 9), NULL, 0, 1, 1, 1, 16, 16, 64, 1.0, w, NULL) == 1
    # a valid window with null pointers is still rejected; empty query is a no-op
    assert lib.fa_forward_window(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 16, 16, 64, 1.0, 4, NULL) == 1
    assert lib.fa_forward_window(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 0, 16, 64, 1.0, 4, NULL) == 0
    assert lib.fa_forward_window(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 16, 16, 96, 1.0, 4, NULL) == 2


def test_decode_window_rejects_bad_window_on_host():
    lib = fa.load_library()
    for w in (0, -1):
        assert lib.fa_decode_splitkv_window(*([NULL] * 6), NULL, 0, 2, 32, 8, 1024, 128, 0.1, 256, w, NULL) == 1
    # otherwise the same checks as fa_decode_splitkv (G = 16 unsupported)
    assert lib.fa_decode_splitkv_window(*([NULL] * 6), NULL, 0, 2, 32, 2, 1024, 128, 0.1, 256, 8, NULL) == 2


def test_context_parallel_decode_argument_checks():
    lib = fa.load_library()
    # partial decode: the same checks as fa_decode_splitkv; a null fp32 output is rejected
    assert lib.fa_decode_splitkv_partial(*([NULL] * 6), NULL, 0, 2, 32, 2, 1024, 128, 0.1, 256, NULL) == 2
    assert lib.fa_decode_splitkv_partial(*([NULL] * 6), NULL, 0, 2, 32, 8, 1024, 128, 0.1, 256, NULL) == 1
    # merge: (o_parts, o_stride, lse_parts, lse_stride, o, lse, R, B, Hq, d, stream)
    assert lib.fa_decode_merge(NULL, 0, NULL, 0, NULL, NULL, 0, 2, 4, 64, NULL) == 1     # R = 0
    assert lib.fa_decode_merge(NULL, 0, NULL, 0, NULL, NULL, 2, 2, 4, 96, NULL) == 2     # head dim
    assert lib.fa_decode_merge(NULL, 0, NULL, 0, NULL, NULL, 2, 0, 4, 64, NULL) == 0     # no rows: no-op
    assert lib.fa_decode_merge(NULL, 0, NULL, 0, NULL, NULL, 2, 2, 4, 64, NULL) == 1     # null pointers
    buf = (ctypes.c_uint8 * 256)()
    base = ctypes.addressof(buf) + (16 - ctypes.addressof(buf) % 16) % 16
    al = ctypes.c_void_p(base)
    rows, d = 2 * 4, 64
    # strides shorter than one partial
    assert lib.fa_decode_merge(al, rows * d - 4, al, rows, al, al, 2, 2, 4, d, NULL) == 1
    assert lib.fa_decode_merge(al, rows * d, al, rows - 1, al, al, 2, 2, 4, d, NULL) == 1
    # O stride not a multiple of 4 floats, or a misaligned O block
    assert lib.fa_decode_merge(al, rows * d + 2, al, rows, al, al, 2, 2, 4, d, NULL) == 3
    assert lib.fa_decode_merge(ctypes.c_void_p(base + 8), rows * d, al, rows, al, al, 2, 2, 4, d, NULL) == 3


def test_fp8_forward_argument_checks():
    lib = fa.load_library()
    args = (1, 1, 1, 16, 16)
    # (q, k, v, q_descale, k_descale, v_descale, o, lse, B, Hq, Hkv, Tq, Tk, d, scale, causal, stream)
    for bad in ((0.0, 1.0, 1.0), (1.0, -1.0, 1.0), (1.0, 1.0, float("inf")), (float("nan"), 1.0, 1.0)):
        assert lib.fa_forward_fp8(NULL, NULL, NULL, *bad, NULL, NULL, *args, 128, 1.0, 0, NULL) == 1
    assert lib.fa_forward_fp8(NULL, NULL, NULL, 1.0, 1.0, 1.0, NULL, NULL, *args, 64, 1.0, 0, NULL) == 2
    assert lib.fa_forward_fp8(NULL, NULL, NULL, 1.0, 1.0, 1.0, NULL, NULL, *args, 128, 1.0, 0, NULL) == 1
    assert lib.fa_forward_fp8(NULL, NULL, NULL, 1.0, 1.0, 1.0, NULL, NULL, 1, 1, 1, 0, 16, 128, 1.0, 0, NULL) == 0


def test_decode_row_limit():
    """One warp per (sequence, head) row in the merge kernels: B * Hq above
    2^26 is rejected on the host."""
    lib = fa.load_library()
    big = (1 << 26) // 32 + 1
    assert lib.fa_decode_splitkv(*([NULL] * 6), NULL, 0, big, 32, 8, 1024, 128, 0.1, 256, NULL) == 1
    assert lib.fa_decode_merge(NULL, 0, NULL, 0, NULL, NULL, 2, big, 32, 128, NULL) == 1


def test_dropout_forward_argument_checks():
    lib = fa.load_library()
    args = (1, 1, 1, 16, 16, 64, 1.0, 0)
    for p in (-0.1, 1.0, 1.5, float("nan")):
        assert lib.fa_forward_dropout(NULL, NULL, NULL, NULL, NULL, *args, p, 1, 0, NULL) == 1
    assert lib.fa_forward_dropout(NULL, NULL, NULL, NULL, NULL, *args, 0.1, 1, 0, NULL) == 1   # null pointers
    assert lib.fa_forward_dropout(NULL, NULL, NULL, NULL, NULL, 1, 1, 1, 16, 16, 96, 1.0, 0, 0.1, 1, 0,
                                  NULL) == 2


def test_header_is_plain_c_and_links(tmp_path):
    """include/fa.h compiles as strict C99 and a C program links against
    libfa.so and calls it (host-side checks only, no GPU)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fa.load_library()
    src = tmp_path / "t.c"
    src.write_text(
        '#include "fa.h"\n#include <string.h>\n'
        "int main(void) {\n"
        '  if (strcmp(fa_status_string(FA_ERR_ALIGNMENT), "FA_ERR_ALIGNMENT")) return 1;\n'
        "  if (fa_forward(0, 0, 0, 0, 0, 1, 1, 1, 16, 16, 96, 1.0f, 0, 0) != FA_ERR_UNSUPPORTED) return 2;\n"
        "  if (fa_decode_workspace_bytes(1, 1, 10, 96, 256) != 0) return 3;\n"
        "  return fa_version() > 0 ? 0 : 4;\n}\n")
    libdir = os.path.dirname(fa.LIB_PATH)
    exe = tmp_path / "t"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", libdir, "-lfa", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_new_entry_points_check_alignment_before_launch():
    lib = fa.load_library()
    buf = (ctypes.c_uint8 * 256)()
    base = ctypes.addressof(buf) + (16 - ctypes.addressof(buf) % 16) % 16
    al, odd = ctypes.c_void_p(base), ctypes.c_void_p(base + 4)
    # dropout forward, misaligned output
    assert lib.fa_forward_dropout(al, al, al, odd, al, 1, 1, 1, 16, 16, 64, 1.0, 0, 0.1, 1, 0, NULL) == 3
    # fp8 forward, misaligned q
    assert lib.fa_forward_fp8(odd, al, al, 1.0, 1.0, 1.0, al, al, 1, 1, 1, 16, 16, 128, 1.0, 0, NULL) == 3
    # partial decode, misaligned fp32 output
    assert lib.fa_decode_splitkv_partial(al, al, al, al, odd, al, al, 1 << 20, 1, 4, 4, 64, 128, 0.1, 256,
                                         NULL) == 3


def test_every_exported_symbol_is_declared():
    """The library exports no fa_* function that include/fa.h does not
    declare (so the header is the whole boundary)."""
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("no nm")
    fa.load_library()
    out = subprocess.run([nm, "-D", "--defined-only", fa.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if ln.split() and ln.split()[-1].startswith("fa_")})
    assert exported == _header_functions()


def test_deterministic_backward_argument_checks():
    lib = fa.load_library()
    args = [NULL] * 9 + [NULL, 0]
    # a window needs causal = 1, and must not be negative
    assert lib.fa_backward_deterministic(*args, 1, 1, 1, 16, 16, 64, 1.0, 0, 8, NULL) == 1
    assert lib.fa_backward_deterministic(*args, 1, 1, 1, 16, 16, 64, 1.0, 1, -1, NULL) == 1
    # the shared prefill checks: GQA divisibility, head size, finite scale
    assert lib.fa_backward_deterministic(*args, 1, 3, 2, 16, 16, 64, 1.0, 1, 0, NULL) == 1
    assert lib.fa_backward_deterministic(*args, 1, 1, 1, 16, 16, 96, 1.0, 1, 0, NULL) == 2
    assert lib.fa_backward_deterministic(*args, 1, 1, 1, 16, 16, 64, float("nan"), 0, 0, NULL) == 1
    # null pointers are rejected; an empty problem is a no-op
    assert lib.fa_backward_deterministic(*args, 1, 1, 1, 16, 16, 64, 1.0, 1, 0, NULL) == 1
    assert lib.fa_backward_deterministic(*args, 0, 1, 1, 16, 16, 64, 1.0, 1, 0, NULL) == 0
