"""Host-side tests of the C ABI (no GPU): the library builds and loads, exports
every entry point include/gdn.h declares, and rejects bad arguments before any
CUDA call."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_gated_quant_b200 import _lib
from nvfp4_w4a4_gated_quant_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(gdn_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    assert set(_lib.EXPORTED) <= set(names)


def test_version_and_status_strings(L):
    assert L.gdn_version().decode().count(".") == 2
    assert L.gdn_status_string(0) == b"ok"
    for s in range(1, 7):
        assert L.gdn_status_string(s) not in (b"ok", b"unknown status")


def test_workspace_queries(L):
    assert L.gdn_quantize_workspace_size() >= 4
    assert L.gdn_scales_tiled_bytes(1, 64) == 128 * 4
    assert L.gdn_scales_tiled_bytes(129, 128) == 256 * 8
    cfg = _lib.layer_cfg(4, 8192, 5120, 32, 128, 128)
    ws = _lib.gdn_layer_workspace_size(cfg)
    offs = _lib.gdn_layer_workspace_offsets(cfg)
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    M = 4 * 8192
    assert offs[_lib.WS_X_SCALES] - offs[_lib.WS_X_CODES] >= M * 5120 // 2
    assert ws >= offs[-1]


def test_bad_arguments_are_rejected_before_launch(L):
    null = None
    # negative rows, bad mode, missing workspace in dynamic mode
    assert L.gdn_quantize_nvfp4(null, 0, -1, 64, 64, 0, null, null, null, 0, 0, ctypes.c_void_p(16), null, 0, null) == 1
    assert L.gdn_quantize_nvfp4(null, 0, 0, 64, 64, 7, null, null, null, 0, 0, ctypes.c_void_p(16), null, 0, null) == 1
    assert L.gdn_quantize_nvfp4(null, 0, 4, 64, 64, 0, null, null, null, 0, 0, ctypes.c_void_p(16), null, 0, null) == 6
    # cols not a multiple of 64 for the tiled layout
    assert L.gdn_quantize_nvfp4(ctypes.c_void_p(256), 0, 4, 48, 48, 1, ctypes.c_void_p(256), ctypes.c_void_p(256),
                                ctypes.c_void_p(256), 0, 0, ctypes.c_void_p(256), null, 0, null) == 2
    # misaligned x
    assert L.gdn_quantize_nvfp4(ctypes.c_void_p(258), 0, 4, 64, 64, 1, ctypes.c_void_p(256), ctypes.c_void_p(256),
                                ctypes.c_void_p(256), 0, 0, ctypes.c_void_p(256), null, 0, null) == 3
    # GEMM: K not a multiple of 64, segments not covering N
    A = _lib.Nvfp4(256, 256)
    seg = (_lib.Segment * 1)()
    seg[0].n_begin, seg[0].n_end, seg[0].kind, seg[0].g_b, seg[0].out, seg[0].ld_out = 0, 8, 0, 256, 256, 8
    assert L.gdn_gemm_nvfp4(ctypes.byref(A), ctypes.c_void_p(256), ctypes.byref(A), 8, 8, 96, seg, 1, null) == 2
    assert L.gdn_gemm_nvfp4(ctypes.byref(A), ctypes.c_void_p(256), ctypes.byref(A), 8, 16, 64, seg, 1, null) == 1
    assert L.gdn_gemm_nvfp4(ctypes.byref(A), ctypes.c_void_p(256), ctypes.byref(A), 8, 8, 64, seg, 9, null) == 1
    # delta rule: unsupported head dims
    assert L.gdn_delta_rule_fwd(null, null, null, 96, 96, 96, null, null, null, 1, 1, 1, 96, 64, 1,
                                null, null, null, 0, null) == 2
    # delta rule step: unknown flag, unsupported head dim, missing output state
    assert L.gdn_delta_rule_step(null, null, null, 128, 128, 128, null, null, null, ctypes.c_void_p(256), 1, 1, 1,
                                 128, 128, 16, null, null) == 1
    assert L.gdn_delta_rule_step(null, null, null, 96, 96, 96, null, null, null, ctypes.c_void_p(256), 1, 1, 1,
                                 96, 64, 1, null, null) == 2
    assert L.gdn_delta_rule_step(null, null, null, 128, 128, 128, null, null, null, null, 1, 0, 1,
                                 128, 128, 1, null, null) == 1
    # watchdog self-test: poll limit out of range
    assert L.gdn_selftest_bounded_wait(0, null) == 1
    # gates: H must be positive
    assert L.gdn_gates(null, null, 4, 0, null, null, null, null, null) == 1
    # layer: workspace missing
    cfg = _lib.layer_cfg(1, 64, 256, 2, 128, 128)
    w = _lib.LayerWeights()
    assert L.gdn_layer_fwd(ctypes.byref(w), ctypes.byref(cfg), null, null, null, null, null, 0, null) == 6


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of the ABI structs have the C compiler's sizes and
    field offsets (a C program including include/gdn.h prints them)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    mirrors = {"gdn_nvfp4_t": _lib.Nvfp4, "gdn_epilogue_segment_t": _lib.Segment,
               "gdn_layer_cfg_t": _lib.LayerCfg, "gdn_layer_weights_t": _lib.LayerWeights}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "gdn.h"', "int main(void) {"]
    for cname, py in mirrors.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in mirrors.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_static_scratch_size_matches_header():
    """The binding's copy of the static scratch size is the header's."""
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    m = re.search(r"#define\s+GDN_LAYER_STATIC_WS_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "GDN_LAYER_STATIC_WS_BYTES not found in gdn.h"
    assert _lib.LAYER_STATIC_WS_BYTES == int(m.group(1)) << int(m.group(2))
