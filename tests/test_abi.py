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

    assert S.lib.stq_abi_version() == 2
    assert S.status_string(-2) == "STQ_ERR_SHAPE"
    for name in declared_functions():
        assert name in S.SIGNATURES, name
    d = S.make_desc(8, 6144, 2048, 256, 8)
    ws = S.moe_workspace_bytes(d)
    # routed h (bf16) + Y (f32) dominate: (P+T)*I*2 + (P+T)*H*4
    assert ws >= (64 + 8) * 2048 * 2 + (64 + 8) * 6144 * 4
    assert S.moe_workspace_bytes(S.make_desc(8, 6144, 2048, 256, 300)) == 0       # k > E
    # the fused RMS normalisation wants a bf16 output and a finite eps >= 0
    assert S.moe_workspace_bytes(S.make_desc(8, 512, 256, 8, 2, norm_eps=1e-6)) > 0
    assert S.moe_workspace_bytes(S.make_desc(8, 512, 256, 8, 2, out_fp32=True, norm_eps=1e-6)) == 0
    assert S.moe_workspace_bytes(S.make_desc(8, 512, 256, 8, 2, norm_eps=-1.0)) == 0
    assert S.moe_workspace_bytes(S.make_desc(8, 512, 256, 8, 2, norm_eps=float("nan"))) == 0
    # T*k < 2^30 keeps pair and row indices (P + T) in int32
    assert S.moe_workspace_bytes(S.make_desc((1 << 27) - 1, 256, 256, 256, 8)) > 0
    assert S.moe_workspace_bytes(S.make_desc(1 << 27, 256, 256, 256, 8)) == 0
    assert S.moe_workspace_bytes(S.make_desc((1 << 31) - 1, 256, 256, 256, 32)) == 0
    # host-side validation returns before any device work (null pointers, bad shapes)
    assert S.lib.stq1_pack(None, 16, 256, None, None, None) == -1
    assert S.lib.stq1_gemv(ctypes.c_void_p(16), 16, 100, ctypes.c_void_p(16), 1, ctypes.c_void_p(16), None) == -2
    assert S.lib.stq1_gemv(ctypes.c_void_p(8), 16, 256, ctypes.c_void_p(16), 1, ctypes.c_void_p(16), None) == -3
    assert S.lib.mxfp8_quantize_bf16(ctypes.c_void_p(16), 4, 48, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == -2


C_LAYOUT = r"""
#include <stddef.h>
#include <stdio.h>
#include "stqmoe.h"
#define F(T, m) printf("%s.%s %zu %zu\n", #T, #m, offsetof(T, m), sizeof(((T*)0)->m))
int main(void) {
  printf("moe_desc %zu\nmoe_weights %zu\n", sizeof(moe_desc), sizeof(moe_weights));
  F(moe_desc, T); F(moe_desc, H); F(moe_desc, I); F(moe_desc, E); F(moe_desc, k);
  F(moe_desc, out_fp32); F(moe_desc, add_residual); F(moe_desc, regime); F(moe_desc, norm_out);
  F(moe_desc, norm_eps);
  F(moe_weights, fmt); F(moe_weights, gate); F(moe_weights, up); F(moe_weights, down);
  F(moe_weights, gate_sc); F(moe_weights, up_sc); F(moe_weights, down_sc);
  F(moe_weights, sh_gate); F(moe_weights, sh_up); F(moe_weights, sh_down); F(moe_weights, sh_fmt);
  F(moe_weights, sh_gate_sc); F(moe_weights, sh_up_sc); F(moe_weights, sh_down_sc);
  return 0;
}
"""


def test_struct_layouts_match_the_header(tmp_path):
    """The binding's ctypes structs have the C header's sizes and field offsets."""
    import bit_quantized_moe_stq1_b200 as S

    src = tmp_path / "layout.c"
    src.write_text(C_LAYOUT)
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    sizes = dict(l.split() for l in lines[:2])
    assert int(sizes["moe_desc"]) == ctypes_size(S.MoeDesc)
    assert int(sizes["moe_weights"]) == ctypes_size(S.MoeWeights)
    for line in lines[2:]:
        if not line:
            continue
        name, off, size = line.split()
        struct, field = name.split(".")
        cls = S.MoeDesc if struct == "moe_desc" else S.MoeWeights
        desc = getattr(cls, field)
        assert (desc.offset, desc.size) == (int(off), int(size)), name


def ctypes_size(cls):
    import ctypes
    return ctypes.sizeof(cls)


def test_moe_host_validation(built):
    """Argument checks of moe_expert_forward and moe_workspace_bytes return before any launch:
    regime and shared-expert format out of range, MXFP8 shared expert without scales or with
    misaligned scales, workspace too small (fake, never dereferenced device pointers)."""
    import ctypes

    import bit_quantized_moe_stq1_b200 as S

    P = ctypes.c_void_p
    fake = P(1 << 20)
    y = P(1 << 21)
    ws = P(1 << 22)

    def call(desc, w, ws_bytes=1 << 40):
        return S.lib.moe_expert_forward(ctypes.byref(desc), fake, fake, fake, ctypes.byref(w), y, ws, ws_bytes, None)

    good = S.make_desc(4, 512, 256, 8, 2)
    assert S.moe_workspace_bytes(good) > 0
    bad_regime = S.make_desc(4, 512, 256, 8, 2, regime=3)
    assert S.moe_workspace_bytes(bad_regime) == 0
    w_stq = S.MoeWeights(S.FMT_STQ1_0, fake, fake, fake, None, None, None, None, None, None, 0, None, None, None)
    assert call(bad_regime, w_stq) == -1  # STQ_ERR_INVALID_ARG
    w_bad_fmt = S.MoeWeights(S.FMT_STQ1_0, fake, fake, fake, None, None, None, fake, fake, fake, 7, None, None, None)
    assert call(good, w_bad_fmt) == -1
    w_no_sc = S.MoeWeights(S.FMT_STQ1_0, fake, fake, fake, None, None, None, fake, fake, fake, S.SHARED_MXFP8,
                           None, None, None)
    assert call(good, w_no_sc) == -1
    w_misaligned = S.MoeWeights(S.FMT_STQ1_0, fake, fake, fake, None, None, None, fake, fake, fake,
                                S.SHARED_MXFP8, P((1 << 20) + 2), fake, fake)
    assert call(good, w_misaligned) == -3  # STQ_ERR_ALIGN
    w_mx8 = S.MoeWeights(S.FMT_STQ1_0, fake, fake, fake, None, None, None, fake, fake, fake, S.SHARED_MXFP8,
                         fake, fake, fake)
    assert call(good, w_mx8, ws_bytes=S.moe_workspace_bytes(good) - 1) == -7  # STQ_ERR_WORKSPACE


def test_workspace_mxfp8_regions_hold_pairs_and_tokens(built):
    """The MXFP8 regions of x and h have rows for the T*k routed pairs and the T tokens of
    the shared expert, in the order the header states."""
    import ctypes

    import bit_quantized_moe_stq1_b200 as S

    T, H, I, E, k = 37, 768, 512, 16, 4
    d = S.make_desc(T, H, I, E, k)
    P = T * k
    off = {r: S.lib.moe_workspace_offset(ctypes.byref(d), i) for i, r in enumerate(S.WS_REGIONS)}
    total = S.moe_workspace_bytes(d)
    ends = sorted(off.values()) + [total]
    room = {r: ends[ends.index(o) + 1] - o for r, o in off.items()}
    assert room["xq"] >= (P + T) * H and room["xs"] >= (P + T) * H // 32
    assert room["hq"] >= (P + T) * I and room["hs"] >= (P + T) * I // 32
    assert room["h"] >= (P + T) * I * 2 and room["Y"] >= (P + T) * H * 4
    assert all(o % 256 == 0 for o in off.values())


def test_timing_kinds_match_the_header():
    """The binding names the timing hook's kernel kinds in the header's enum order."""
    import bit_quantized_moe_stq1_b200 as S

    text = open(os.path.join(ROOT, "include", "stqmoe.h")).read()
    body = re.search(r"enum\s*\{\s*(STQ_K_ROUTER_LOGITS[^}]*)\}", text).group(1)
    names = [n.strip().split("=")[0].strip() for n in body.split(",") if n.strip()]
    assert names[-1] == "STQ_K_COUNT"
    expect = [n[len("STQ_K_"):].lower() for n in names[:-1]]
    assert expect == list(S.KERNEL_KINDS)
    # the library's own names (also its NVTX range names) agree
    assert [S.lib.stq_kernel_kind_name(i).decode() for i in range(len(expect))] == expect
    assert S.lib.stq_kernel_kind_name(len(expect)).decode() == "unknown"
    assert S.lib.stq_kernel_kind_name(-1).decode() == "unknown"
