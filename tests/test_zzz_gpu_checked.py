"""The checked build on the GPU: small STQ1_0 decode and prefill layers and an MXFP4 layer,
each with a BF16 shared expert, run through libstqmoe_checked.so (STQMOE_CHECKED=1) give
bit-identical outputs to the default library and a clear error word: its index re-checks
change no arithmetic.  Both builds run in subprocesses of the same script.  Collected
after the other GPU tests."""

import importlib.util
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import numpy as np
import torch
import bit_quantized_moe_stq1_b200 as S
import workloads as W

assert S.lib.stq_checked_build() == int(sys.argv[1])
dev = "cuda"
H, I = 512, 256
out = {}
cases = {"decode": (5, "stq", S.REGIME_DECODE), "prefill": (300, "stq", S.REGIME_PREFILL),
         "mx": (40, "mx", S.REGIME_AUTO)}
for name, (T, fmt, regime) in cases.items():
    E, k, tag = 8, 2, ("checked-build", name)
    shapes = (("g", I, H), ("u", I, H), ("d", H, I))
    if fmt == "stq":
        mats = [S.stq1_pack(W.stq_grid_weights(E * r, c, dev, 0, tag, w)) for w, r, c in shapes]
        routed = (S.FMT_STQ1_0, *mats, None, None, None)
    else:
        q = [W.mxfp4_random(E * r, c, dev, 0, tag, w) for w, r, c in shapes]
        routed = (S.FMT_MXFP4, q[0][0], q[1][0], q[2][0], q[0][1], q[1][1], q[2][1])
    sh = [W.bf16_normal((r, c), 0.02, dev, 0, tag, "s" + w) for w, r, c in shapes]
    x = W.bf16_normal((T, H), 1.0, dev, 0, tag, "x")
    ids, tw = W.zipf_routing(T, E, k, dev, 0, tag, "ids")
    desc = S.make_desc(T, H, I, E, k, out_fp32=True, regime=regime)
    ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=dev)
    y = torch.empty((T, H), dtype=torch.float32, device=dev)
    S.moe_expert_forward(desc, x, ids, tw, S.ExpertWeights(*routed, *sh), y, ws)
    out[name + "_err"] = np.array([S.moe_get_device_error(ws)])
    out[name] = y.cpu().numpy()
np.savez(sys.argv[2], **out)
"""


def test_checked_build_matches_the_default_build(tmp_path):
    # the default library is the one this process has loaded; only the checked one may
    # need building here (nvcc is on the box), and building it touches nothing else
    spec = importlib.util.spec_from_file_location("_stq_build", os.path.join(ROOT, "bit_quantized_moe_stq1_b200",
                                                                             "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    if not os.path.exists(b.CHECKED_LIB):
        b.build(checked=True)
    outs = []
    for checked in (0, 1):
        path = str(tmp_path / f"out{checked}.npz")
        env = dict(os.environ, STQMOE_CHECKED=str(checked))
        res = subprocess.run([sys.executable, "-c", SCRIPT, str(checked), path], cwd=ROOT, env=env,
                             capture_output=True, text=True, timeout=900)
        assert res.returncode == 0, res.stderr[-3000:]
        outs.append(np.load(path))
    assert sorted(outs[0].files) == sorted(outs[1].files)
    for key in outs[0].files:
        assert np.array_equal(outs[0][key], outs[1][key]), key
    for name in ("decode", "prefill", "mx"):
        assert int(outs[1][name + "_err"][0]) == 0, name
