"""The benchmark's oracle arm (`bench.py --impl reference`) runs on the CPU alone: it never
imports the CUDA package, prints the same `config` as the GPU arm and a finite
`ms_per_step`, and states the host cores its sample used."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROBE = r"""
import json, sys, types
sys.path.insert(0, {root!r})
import bench
args = types.SimpleNamespace(workload={wl!r}, steps=1, warmup=3, gpus=1, experts=256)
bench.run_reference(args)
print(json.dumps({{"loaded": sorted(m for m in sys.modules if m.startswith("bit_quantized_moe_stq1_b200")),
                   "config": bench.base_config({wl!r}, 1)}}))
"""


def _run(wl):
    out = subprocess.run([sys.executable, "-c", PROBE.format(root=ROOT, wl=wl)], capture_output=True, text=True,
                         timeout=600, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(l) for l in out.stdout.strip().splitlines() if l.startswith("{")]
    return lines[-2], lines[-1]


def test_reference_arm_is_cpu_only_and_matches_config():
    line, probe = _run("stq_matvec")
    assert probe["loaded"] == []
    assert line["impl"] == "reference" and line["config"] == probe["config"]
    assert line["ms_per_step"] > 0 and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
