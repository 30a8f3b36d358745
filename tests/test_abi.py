"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
symbol include/*.h declares (no compute calls here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[\w\s\*]+?\b(zo_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def built_lib():
    from zeroth_order_fine_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_every_declared_symbol_is_exported(built_lib):
    names = declared_functions()
    assert len(names) >= 20
    missing = [n for n in sorted(names) if not hasattr(built_lib, n)]
    assert not missing, missing


def test_binding_covers_the_header():
    from zeroth_order_fine_b200 import zo
    assert declared_functions() <= set(zo.EXPORTED)


def test_struct_sizes_match_header(built_lib):
    """The ctypes mirrors have the C layouts (checked against offsets fixed by the header)."""
    from zeroth_order_fine_b200 import zo
    assert ctypes.sizeof(zo.zo_model_desc) == 13 * 4
    assert ctypes.sizeof(zo.zo_targets) == 24
    assert zo.zo_options.stream.offset == 64 and ctypes.sizeof(zo.zo_options) == 88   # 84 bytes of fields, 8-aligned
    assert ctypes.sizeof(zo.zo_layer_weights) == 20 * 8


def test_struct_layouts_match_the_c_compiler(tmp_path):
    """sizeof/offsetof of every ABI struct from gcc on include/zo.h equal the ctypes mirrors."""
    import os
    import shutil
    import subprocess
    from zeroth_order_fine_b200 import zo
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    structs = {"zo_model_desc": zo.zo_model_desc, "zo_layer_weights": zo.zo_layer_weights,
               "zo_weights": zo.zo_weights, "zo_targets": zo.zo_targets,
               "zo_options": zo.zo_options, "zo_stats_t": zo.zo_stats_t}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "zo.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'printf("{name} %zu\\n", sizeof({name}));')
        for f, _ in cls._fields_:
            lines.append(f'printf("{name}.{f} %zu\\n", offsetof({name}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", inc, str(src), "-o", str(exe)], check=True)
    got = dict(l.rsplit(" ", 1) for l in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    for name, cls in structs.items():
        assert int(got[name]) == ctypes.sizeof(cls), name
        for f, _ in cls._fields_:
            assert int(got[f"{name}.{f}"]) == getattr(cls, f).offset, f"{name}.{f}"


def test_library_refuses_bad_create_without_gpu(built_lib):
    """Argument checks run on the host before any CUDA call."""
    from zeroth_order_fine_b200 import zo
    L = zo.lib()
    out = ctypes.c_void_p()
    assert L.zo_create(None, None, None, ctypes.byref(out)) == zo.ZO_ERR_ARG
    assert L.zo_last_error(None)


def test_product_path_does_not_import_oracle():
    for f in glob.glob(os.path.join(ROOT, "zeroth_order_fine_b200", "**", "*.*"), recursive=True):
        if f.endswith((".py", ".cu", ".cpp", ".cuh", ".h")):
            txt = open(f).read()
            assert "import oracle" not in txt and "from oracle" not in txt, f


def test_decode_linear_argument_checks_without_gpu(built_lib):
    """zo_op_linear_decode validates sizes, pointers and the workspace on the host, before
    any CUDA call (placeholder addresses are never dereferenced on these paths)."""
    from zeroth_order_fine_b200 import zo
    L = zo.lib()
    p = ctypes.c_void_p(0x10000)
    call = lambda x, W, y, M, N, K, act, acc, ws, n: L.zo_op_linear_decode(
        x, W, None, y, M, N, K, act, acc, ws, n, None)
    assert call(p, p, p, -1, 256, 64, 0, 0, p, 1 << 20) == zo.ZO_ERR_ARG      # negative M
    assert call(p, p, p, 4, 0, 64, 0, 0, p, 1 << 20) == zo.ZO_ERR_ARG         # empty N
    assert call(p, p, p, 4, 256, 64, 2, 0, p, 1 << 20) == zo.ZO_ERR_ARG       # unknown act
    assert call(p, p, p, 4, 256, 64, 1, 1, p, 1 << 20) == zo.ZO_ERR_ARG       # ReLU + accumulate
    assert call(None, None, None, 0, 256, 64, 0, 0, None, 0) == zo.ZO_OK       # M = 0: no-op
    assert call(None, p, p, 4, 256, 64, 0, 0, p, 1 << 20) == zo.ZO_ERR_ARG    # NULL x
    assert call(p, p, p, 4, 256, 64, 0, 0, None, 1 << 20) == zo.ZO_ERR_ARG    # NULL workspace
    assert call(p, p, p, 4, 256, 64, 0, 0, p, 4 * 256 - 1) == zo.ZO_ERR_ARG   # < one slice
    assert call(p, p, p, 4, 256, 60, 0, 0, p, 1 << 20) == zo.ZO_ERR_UNSUPPORTED  # K % 8
    assert call(p, p, p, 4, 258, 64, 0, 0, p, 1 << 20) == zo.ZO_ERR_UNSUPPORTED  # N % 4


def test_op_error_text_is_empty_before_any_failure(built_lib):
    built_lib.zo_op_last_error.restype = ctypes.c_char_p
    assert built_lib.zo_op_last_error() == b""


def test_debug_build_exports_the_same_symbols_and_says_so(built_lib):
    """libzo_b200_debug.so (ZO_DEBUG: device bounds checks) links from the same sources:
    every declared symbol is there, and zo_debug_build tells the two builds apart."""
    from zeroth_order_fine_b200 import build
    dbg = ctypes.CDLL(build.build(debug=True))
    missing = [n for n in sorted(declared_functions()) if not hasattr(dbg, n)]
    assert not missing, missing
    assert dbg.zo_debug_build() == 1 and built_lib.zo_debug_build() == 0


def test_op_wrappers_refuse_host_tensors_before_any_launch():
    """The ops take raw device pointers: host tensors (or wrong shapes / dtypes) are refused
    in the binding, so nothing reaches a kernel."""
    import torch
    from zeroth_order_fine_b200 import zo
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    W = torch.zeros(32, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        zo.zo_op_linear(x, W)
    with pytest.raises(ValueError, match="CUDA"):
        zo.zo_op_linear_decode(x, W)
    with pytest.raises(ValueError, match="CUDA"):
        zo.zo_op_lm_head_logprob(x, W, torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        zo.zo_op_attention(torch.zeros(10, 3 * 128, dtype=torch.bfloat16), [10], 1, 1, 128)
    with pytest.raises(ValueError, match="CUDA"):
        zo.zo_op_quantize_rows_e4m3(x)
