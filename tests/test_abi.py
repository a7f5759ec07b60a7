"""The C-ABI library loads and exports every function include/*.h declares
(no compute calls: this runs without a GPU)."""

import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "bit_quantized_moe_stq1_b200", "libstqmoe.so")


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def built():
    if not os.path.exists(LIB):
        subprocess.run(["python", os.path.join(ROOT, "bit_quantized_moe_stq1_b200", "build.py")], check=True)
    return LIB


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["stq1_pack", "stq1_unpack", "mxfp4_pack", "mxfp4_unpack", "mxfp8_quantize_bf16", "stq1_gemv",
              "w4a8_gemm", "moe_router_topk", "moe_permute", "moe_workspace_bytes", "moe_expert_forward",
              "moe_get_device_error", "stq_status_string", "stq_read_error", "stq_abi_version"]:
        assert n in names, n


def test_library_exports_every_declared_symbol(built):
    out = subprocess.run(["nm", "-D", "--defined-only", built], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = declared_functions() - exported
    assert not missing, missing


def test_binding_loads_and_host_side_calls(built):
    import ctypes

    import bit_quantized_moe_stq1_b200 as S

    assert S.lib.stq_abi_version() == 1
    assert S.status_string(-2) == "STQ_ERR_SHAPE"
    for name in declared_functions():
        assert name in S.SIGNATURES, name
    d = S.make_desc(8, 6144, 2048, 256, 8)
    ws = S.moe_workspace_bytes(d)
    # routed h (bf16) + Y (f32) dominate: (P+T)*I*2 + (P+T)*H*4
    assert ws >= (64 + 8) * 2048 * 2 + (64 + 8) * 6144 * 4
    assert S.moe_workspace_bytes(S.make_desc(8, 6144, 2048, 256, 300)) == 0       # k > E
    # host-side validation returns before any device work (null pointers, bad shapes)
    assert S.lib.stq1_pack(None, 16, 256, None, None, None) == -1
    assert S.lib.stq1_gemv(ctypes.c_void_p(16), 16, 100, ctypes.c_void_p(16), 1, ctypes.c_void_p(16), None) == -2
    assert S.lib.stq1_gemv(ctypes.c_void_p(8), 16, 256, ctypes.c_void_p(16), 1, ctypes.c_void_p(16), None) == -3
    assert S.lib.mxfp8_quantize_bf16(ctypes.c_void_p(16), 4, 48, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == -2
