"""The C-ABI library builds, loads and exports every entry point of include/metis.h.

No compute call is made here (these run without a GPU).  The ctypes mirror of
every struct is checked field by field against offsets that gcc computes from
the header itself.
"""

import ctypes
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "metis.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(metis_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(metis_lib):
    names = _declared_functions()
    assert len(names) >= 14
    lib = ctypes.CDLL(metis_lib.LIB_PATH)
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(metis_lib.EXPORTED) == names


def test_status_strings(metis_lib):
    for code in range(7):
        assert metis_lib.status_str(code)
    assert metis_lib.status_str(4) == "device is not sm_100 (B200)"


def test_size_helpers(metis_lib):
    assert metis_lib._codes_bytes(128, 256) == 128 * 128
    assert metis_lib._scales_bytes(128, 256) == 2048
    assert metis_lib._scales_bytes(256, 4096) == 2 * 64 * 512


def test_create_without_gpu_fails_cleanly(metis_lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    handle = ctypes.c_void_p()
    st = metis_lib._create(0, None, ctypes.byref(handle))
    assert st != 0 and not handle.value


def _c_offsets(tmp_path):
    structs = {
        "metis_matrix": ["data", "rows", "cols", "ld"],
        "metis_nvfp4": ["codes", "scales", "tensor_scale", "outer", "inner"],
        "metis_factors": ["rows", "cols", "k", "V", "U", "S", "Uq", "Vq", "sampled_rows", "omega"],
        "metis_decomp_params": ["k", "s", "l_k", "seed", "operand_id", "rounding"],
        "metis_quant_params": ["rounding", "seed", "operand_id", "step", "tensor_scale"],
        "metis_operand": ["rowwise", "colwise", "f"],
    }
    lines = ['#include <stdio.h>', '#include <stddef.h>', f'#include "{HEADER}"', "int main(void) {"]
    for s, fields in structs.items():
        lines.append(f'printf("{s} size %zu\\n", sizeof({s}));')
        for f in fields:
            lines.append(f'printf("{s} {f} %zu\\n", offsetof({s}, {f}));')
    lines.append("return 0; }")
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    res = {}
    for line in out.splitlines():
        s, f, v = line.split()
        res[(s, f)] = int(v)
    return res


def test_ctypes_layout_matches_header(metis_lib, tmp_path):
    off = _c_offsets(tmp_path)
    mirror = {"metis_matrix": metis_lib.Matrix, "metis_nvfp4": metis_lib.Nvfp4Struct,
              "metis_factors": metis_lib.FactorsStruct, "metis_decomp_params": metis_lib.DecompParams,
              "metis_quant_params": metis_lib.QuantParams, "metis_operand": metis_lib.OperandStruct}
    for cname, cls in mirror.items():
        assert ctypes.sizeof(cls) == off[(cname, "size")], cname
        for fname, _ in cls._fields_:
            assert getattr(cls, fname).offset == off[(cname, fname)], (cname, fname)
