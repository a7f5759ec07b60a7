"""The checked build (-DSTQ_CHECKED=1, libstqmoe_checked.so) without a GPU: it compiles,
exports the same C ABI as the default library, reports itself through
stq_checked_build(), and STQMOE_CHECKED=1 makes the binding load it."""

import importlib.util
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _builder():
    spec = importlib.util.spec_from_file_location("_stq_build", os.path.join(ROOT, "bit_quantized_moe_stq1_b200",
                                                                             "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True, check=True).stdout
    return {line.split()[-1] for line in out.splitlines() if " T " in line}


def test_checked_build_has_the_same_abi():
    import bit_quantized_moe_stq1_b200 as S

    b = _builder()
    default, checked = S.LIB_PATH, b.build(checked=True)  # the loaded library is not rebuilt here
    assert os.path.basename(default) == ("libstqmoe_checked.so" if S.CHECKED else "libstqmoe.so")
    assert os.path.basename(checked) == "libstqmoe_checked.so"
    api = set(S.SIGNATURES)
    assert api <= _exported(default) and api <= _exported(checked)
    assert S.lib.stq_checked_build() == (1 if S.CHECKED else 0)


def test_environment_selects_the_checked_library():
    _builder().build(checked=True)
    code = ("import bit_quantized_moe_stq1_b200 as S; "
            "assert S.LIB_PATH.endswith('libstqmoe_checked.so'); assert S.lib.stq_checked_build() == 1")
    env = dict(os.environ, STQMOE_CHECKED="1")
    res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
