"""Benchmark of the routed-expert FFN hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path of the workload over one batch of
synthetic inputs (router, grouping, expert GEMVs with SwiGLU, shared expert,
combine; layer after layer for the stacked workload).  Inputs are resident in
HBM before timing; each step uses a different token batch (rotating over 8) and
the per-step expert weights exceed L2, so no step is served from L2.
Rank 0 prints one JSON line.  Under torchrun every rank runs its own replica
(weak scaling, no collective on the data path); the reported time is the max
over ranks.

--impl reference times the CPU oracle (the plain float64 numpy reference under
oracle/) on a bounded sample of the same workload, on rank 0 only.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "decode_stq"
N_BATCHES = 8
STQ_MAT = 2048 * 6144 // 256 * 42          # 2,064,384 bytes per STQ1_0 expert matrix
STQ_EXPERT = 3 * STQ_MAT                    # 6,193,152
BF16_MAT = 2048 * 6144 * 2                  # 25,165,824
ROUTER_BYTES = 256 * 6144 * 2               # 3,145,728


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, src="fallback")


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.f.flush()
        rows = [l.split(",") for l in open(self.f.name).read().strip().splitlines() if l.count(",") >= 8]
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- workloads


class DecodeSTQ:
    """Decode MoE layer, STQ1_0 experts: 8 BF16 tokens, BF16 router (softmax, top-8,
    renormalised), 256 experts of 6144 -> 2048 -> 6144, one BF16 shared expert."""

    name = "decode_stq"
    unit = "tokens/s"

    def __init__(self, S, dev, tokens=8, layers=1):
        self.S, self.dev = S, dev
        self.wl = W.WORKLOADS["decode_stq"]
        self.T, self.H, self.I, self.E, self.k = tokens, self.wl.H, self.wl.I, self.wl.E, self.wl.k
        self.layers = [self._layer(l) for l in range(layers)]
        self.x = [W.bf16_normal((self.T, self.H), 1.0, dev, 0, "x", b) for b in range(N_BATCHES)]
        self.desc = S.make_desc(self.T, self.H, self.I, self.E, self.k)
        self.ws = torch.zeros(S.moe_workspace_bytes(self.desc), dtype=torch.uint8, device=dev)
        self.y = torch.empty((self.T, self.H), dtype=torch.bfloat16, device=dev)
        self.logits = torch.empty((self.T, self.E), dtype=torch.float32, device=dev)
        self.ids = torch.empty((self.T, self.k), dtype=torch.int32, device=dev)
        self.tw = torch.empty((self.T, self.k), dtype=torch.float32, device=dev)

    def _stq_matrices(self, l, which, rows, cols):
        """E STQ1_0 matrices [rows, cols], packed on the device in chunks of 16 experts."""
        S, E = self.S, self.E
        out = torch.empty(E * rows * cols // 256 * 42, dtype=torch.uint8, device=self.dev)
        per = rows * cols // 256 * 42
        for e0 in range(0, E, 16):
            wf = W.stq_grid_weights(16 * rows, cols, self.dev, 0, "L", l, which, e0)
            S.stq1_pack(wf, out=out[e0 * per:(e0 + 16) * per])
            del wf
        return out

    def _layer(self, l):
        S = self.S
        g = self._stq_matrices(l, "g", self.I, self.H)
        u = self._stq_matrices(l, "u", self.I, self.H)
        d = self._stq_matrices(l, "d", self.H, self.I)
        sh = [W.bf16_normal((self.I, self.H), 0.02, self.dev, 0, "L", l, "sg"),
              W.bf16_normal((self.I, self.H), 0.02, self.dev, 0, "L", l, "su"),
              W.bf16_normal((self.H, self.I), 0.02, self.dev, 0, "L", l, "sd")]
        wr = W.bf16_normal((self.E, self.H), 0.02, self.dev, 0, "L", l, "router")
        return dict(w=S.ExpertWeights(S.FMT_STQ1_0, g, u, d, sh_gate=sh[0], sh_up=sh[1], sh_down=sh[2]), wr=wr)

    def step(self, b, x=None, y=None):
        S = self.S
        x = self.x[b % N_BATCHES] if x is None else x
        y = self.y if y is None else y
        for L in self.layers:
            S.moe_router_topk(x, L["wr"], self.k, self.logits, self.ids, self.tw)
            S.moe_expert_forward(self.desc, x, self.ids, self.tw, L["w"], y, self.ws)
        return y

    def tokens_per_step(self):
        return self.T

    def touched(self, b):
        """Realised number of touched experts per layer for batch b (host bookkeeping)."""
        S = self.S
        out = []
        for L in self.layers:
            ids, _, _ = S.moe_router_topk(self.x[b % N_BATCHES], L["wr"], self.k)
            out.append(int(torch.unique(ids).numel()))
        return out

    def algorithmic_bytes(self, b):
        """Bytes a step must move: touched experts' packed matrices, the shared
        expert, the router, and the activations (x in, y out)."""
        n = self.touched(b)
        per_layer = [t * STQ_EXPERT + 3 * BF16_MAT + ROUTER_BYTES + self.T * self.H * 4 for t in n]
        gate_up = [t * 2 * STQ_MAT + 2 * BF16_MAT + self.T * self.H * 2 + (self.T * self.k + self.T) * self.I * 2
                   for t in n]
        return sum(per_layer), dict(gate_up=gate_up)

    def h2d_d2h(self):
        return self.T * self.H * 2, self.T * self.H * 2


class StqMatvec:
    """One STQ1_0 matrix 2048 x 6144 times one BF16 N(0,1) vector, FP32 out.  The
    2 MB matrix fits in L2, so steps rotate over copies totalling 4x the L2 size."""

    name = "stq_matvec"
    unit = "GB/s"

    def __init__(self, S, dev):
        self.S, self.dev = S, dev
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.ncopies = max(8, int(4 * l2 // STQ_MAT) + 1)
        wf = W.stq_grid_weights(2048, 6144, dev, 0, "mv")
        base = S.stq1_pack(wf)
        self.W = [base.clone() for _ in range(self.ncopies)]
        self.x = [W.bf16_normal((1, 6144), 1.0, dev, 0, "mvx", b) for b in range(N_BATCHES)]
        self.y = torch.empty((1, 2048), dtype=torch.float32, device=dev)

    def step(self, b, x=None, y=None):
        x = self.x[b % N_BATCHES] if x is None else x
        return self.S.stq1_gemv(self.W[b % self.ncopies], 2048, 6144, x, self.y if y is None else y)

    def tokens_per_step(self):
        return 1

    def algorithmic_bytes(self, b):
        nb = STQ_MAT + 6144 * 2 + 2048 * 4
        return nb, dict(gemv=[nb])

    def h2d_d2h(self):
        return 6144 * 2, 2048 * 4


WORKLOADS = {"decode_stq": DecodeSTQ, "stq_matvec": StqMatvec}


# ----------------------------------------------------------------------------- measurement


def timed_steps(wl, steps, warmup, dist):
    torch.cuda.synchronize()
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        wl.step(warmup + i)
    stop.record()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    return start.elapsed_time(stop)


def kernel_times(S, wl, steps, warmup):
    """Per-kernel CUDA-event durations over `steps` steps (events recorded by the
    library on the launching stream)."""
    timer = S.KernelTimer(capacity=4096)
    per_kind = {}
    for i in range(steps):
        with timer:
            wl.step(warmup + i)
        for kind, ms in timer.results():
            per_kind.setdefault(kind, []).append(ms)
    return per_kind


def e2e_steps(wl, steps, warmup):
    """Same metric end to end through the public API with pinned host buffers:
    H2D of the step's tokens and D2H of its output inside the timed region."""
    x_dev = wl.x[0]
    hx = [wl.x[b].cpu().pin_memory() for b in range(N_BATCHES)]
    y_dev = torch.empty_like(wl.y)
    hy = torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory()
    for i in range(warmup):
        x_dev.copy_(hx[i % N_BATCHES], non_blocking=True)
        wl.step(i, x=x_dev, y=y_dev)
        hy.copy_(y_dev, non_blocking=True)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    xs = torch.empty_like(x_dev)
    start.record()
    for i in range(steps):
        xs.copy_(hx[(warmup + i) % N_BATCHES], non_blocking=True)
        wl.step(warmup + i, x=xs, y=y_dev)
        hy.copy_(y_dev, non_blocking=True)
    stop.record()
    torch.cuda.synchronize()
    return start.elapsed_time(stop)


def run_ours(args):
    dist = int(os.environ.get("WORLD_SIZE", "1")) > 1
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if dist:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import bit_quantized_moe_stq1_b200 as S

    wl = WORKLOADS[args.workload](S, dev)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed_steps(wl, args.steps, args.warmup, dist)
    clocks = clk.summary()
    ms_t = torch.tensor([ms], device=dev)
    if dist:
        torch.distributed.all_reduce(ms_t, op=torch.distributed.ReduceOp.MAX)
    ms = float(ms_t.item())
    n = int(os.environ.get("WORLD_SIZE", "1"))
    ms_step = ms / args.steps
    kt = kernel_times(S, wl, args.steps, args.warmup)
    e2e_ms = e2e_steps(wl, args.steps, args.warmup)
    ab, per_kernel_bytes = wl.algorithmic_bytes(0)
    pk = peaks()
    # dominant kernel: the kind with the largest total time
    tot = {k: sum(v) for k, v in kt.items()}
    dom = max(tot, key=tot.get)
    launches = len(kt[dom])
    avg_ms = tot[dom] / launches
    kb = per_kernel_bytes.get(dom)
    kb_launch = float(np.mean(kb)) if kb else None
    achieved = kb_launch / (avg_ms * 1e-3) / 1e9 if kb_launch else None
    tps = wl.tokens_per_step()
    gpu_launches = sum(len(v) for v in kt.values())
    if wl.unit == "GB/s":
        value = n * ab / (ms_step * 1e-3) / 1e9
        metric = "STQ1_0 matvec achieved HBM GB/s (2048x6144, 1 token)"
        e2e_val = n * ab / (e2e_ms / args.steps * 1e-3) / 1e9
    else:
        value = n * tps / (ms_step * 1e-3)
        metric = "MoE-layer tokens/s"
        e2e_val = n * tps / (e2e_ms / args.steps * 1e-3)
    h2d, d2h = wl.h2d_d2h()
    out = {
        "metric": metric, "value": value, "unit": wl.unit, "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 activations x packed STQ1_0 weights, fp32 accumulate",
        "data": "synthetic (seeded generators; random weights on the format grids)",
        "config": {"workload": wl.name, "tokens_per_step": tps, "hbm_bytes_per_step": ab,
                   "l2": "weights per step exceed L2; token batches rotate over 8",
                   "parallelism": f"replicas x{n}"},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                     "frac": (achieved / pk["hbm"]) if achieved else None, "peak_source": pk["src"],
                     "traffic": None, "bytes_per_launch": kb_launch, "avg_launch_ms": avg_ms},
        "kernels_ms": {k: statistics.mean(v) for k, v in kt.items()},
        "gpu_launches": gpu_launches,
        "e2e": {"value": e2e_val, "unit": wl.unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }
    if rank == 0 and not dist:
        out["cpu_baseline"] = cpu_baseline(wl, dev)
    elif rank == 0:
        out["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(out))
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------------------------- oracle timing


def _oracle_decode_token(wl, dev, b=0, t=0):
    """The oracle's layer for one token: router, its top-8 experts and the shared
    expert, from the generator's tensors (weights decoded from the oracle's own
    packing of the generator's grid values)."""
    from oracle import formats as F
    from oracle import moe as M

    x = wl.x[b][t:t + 1]
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16)
    L = 0
    wr = wl.layers[L]["wr"].view(torch.int16).cpu().numpy().view(np.uint16)
    ids, w, _ = M.router_topk(xb, wr, wl.k)
    X = F.bf16_decode(xb)
    y = np.zeros((1, wl.H))
    for s, e in enumerate(ids[0]):
        mats = []
        for which, (rows, cols) in (("g", (wl.I, wl.H)), ("u", (wl.I, wl.H)), ("d", (wl.H, wl.I))):
            e0 = (int(e) // 16) * 16
            wf = W.stq_grid_weights(16 * rows, cols, dev, 0, "L", L, which, e0)
            blk = wf[(int(e) - e0) * rows:(int(e) - e0 + 1) * rows].cpu().numpy()
            mats.append(F.stq1_unpack(F.stq1_pack(blk), rows, cols))
        out = M.expert_ffn_bf16h(mats[0], mats[1], mats[2], X)
        y += w[0, s] * out["y"]
    sh = [wl.layers[L]["w"].sh_gate, wl.layers[L]["w"].sh_up, wl.layers[L]["w"].sh_down]
    out = M.expert_ffn_bf16h(*[m.float().double().cpu().numpy() for m in sh], X)
    return y + out["y"]


def cpu_baseline(wl, dev):
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        if wl.name == "stq_matvec":
            from oracle import moe as M
            Wb = wl.W[0].cpu().numpy()
            xb = wl.x[0].view(torch.int16).cpu().numpy().view(np.uint16)
            reps = 0
            while time.perf_counter() - t0 < 10.0:
                M.stq1_gemv(Wb, 2048, 6144, xb)
                reps += 1
            dt = time.perf_counter() - t0
            return {"value": reps * (STQ_MAT + 6144 * 2 + 2048 * 4) / dt / 1e9, "unit": "GB/s", "cores": 1,
                    "kind": "oracle", "sample": f"{reps} full matvecs (unpack + float64 matvec)"}
        _oracle_decode_token(wl, dev)
        dt = time.perf_counter() - t0
    return {"value": 1.0 / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "1 token of one layer: router, its 8 experts (unpack + float64 FFN) and the shared expert"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    import bit_quantized_moe_stq1_b200 as S

    wl = WORKLOADS[args.workload](S, dev)
    times = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(wl, dev)
        if i >= args.warmup:
            times.append(cb["value"])
    value = statistics.mean(times)
    out = {"impl": "reference", "metric": "MoE-layer tokens/s" if wl.unit != "GB/s" else
           "STQ1_0 matvec achieved HBM GB/s (2048x6144, 1 token)", "value": value, "unit": wl.unit, "n_gpus": 0,
           "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": {"workload": wl.name},
           "cpu_baseline": {"value": value, "unit": wl.unit, "cores": cb["cores"], "kind": "oracle",
                            "sample": cb["sample"]},
           "e2e": {"value": value, "unit": wl.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
