"""Benchmark of the routed-expert FFN hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path of the workload over one batch of
synthetic inputs: router, grouping, activation quantisation (MXFP4 layers),
expert gate/up with fused SwiGLU, down, shared expert and combine, layer after
layer for the stacked workload.  Inputs are resident in HBM before timing; steps
rotate over 8 token batches (and, for the single-matrix workloads, over weight
copies totalling more than 4x L2), so no step is served from L2.  The timed
region replays one CUDA graph per step.  Per-kernel times come from CUDA events
the library records around each launch (captured into the graphs as event
nodes), on the launching stream.  Rank 0 prints one JSON line.  Under torchrun
every rank runs its own replica (weak scaling, no collective on the data path);
the reported time is the max over ranks.

--impl reference times the CPU oracle (the plain float64 numpy reference under
oracle/) on a bounded sample of the same workload, on rank 0 only.
"""

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "stacked_decode"
N_BATCHES = 8
H, I, E, K_TOP = W.HIDDEN, W.INTER, W.EXPERTS, W.TOPK
STQ_MAT = I * H // 256 * 42                 # 2,064,384 bytes per STQ1_0 expert matrix
MX_MAT = I * H // 2 + I * H // 32           # 6,684,672 bytes per MXFP4 matrix (codes + scales)
BF16_MAT = I * H * 2                        # 25,165,824
MX8_MAT = I * H + I * H // 32               # 12,976,128 per MXFP8 matrix (codes + scales)
ROUTER_BYTES = E * H * 2                    # 3,145,728
NOMINAL_FP8_OVER_BF16 = 2.0                 # dense FP8 (kind::mxf8f6f4) / dense BF16 tensor rate
# A second tensor peak for the block-scaled GEMMs: back-to-back tcgen05 kind::mxf8f6f4 MMAs
# (M = 128, N >= 128, one CTA per SM, no memory traffic) measured 8,190 MACs per clock per
# SM on this machine's B200s; at the 1965 MHz maximum SM clock of 148 SMs that is 4.76 PFLOP/s.
MMA_MICROBENCH_TFLOPS = 2 * 8190 * 148 * 1.965e9 / 1e12

# DRAM bytes (read + write) per touched expert of one decode-size launch, from one ncu
# capture of the same kernel build on a smaller case (named profile under profiles/); a
# launch's traffic grows with its touched experts, so the full launch's traffic is this
# figure times its touched experts.  An entry is removed when its kernel changes.
MEASURED_TRAFFIC_PER_EXPERT = {"gate_up_mx": (860.83e6 + 3.90e6) / 64}  # decode_mx, 64 experts, 64 touched
# DRAM bytes (read + write) of one full-size launch, from an ncu capture of the same workload
# and kernel build; an entry is removed when its kernel changes.
MEASURED_TRAFFIC_PER_LAUNCH = {("stq_matvec", "gemv"): 2.09e6, ("w4a8_gemm", "gemm"): 7.54e6,
                               ("stq_pack_ls", "pack_ls"): 50.40e6 + 9.47e3,
                               ("decode_stq", "gate_up"): 286.006528e6 + 1.105152e6,
                               ("prefill_w4a8", "gate_up_mx"): 3.74e9 + 69.87e6,
                               ("prefill_stq", "gate_up_stq_tc"): 1.60e9 + 63.20e6}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """NVML sampling of SM clocks and throttle reasons while the timed region runs."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu, self.samples, self.stop = gpu_index, [], threading.Event()
        self.max_mhz = None

    def _run(self):
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        while not self.stop.is_set():
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            self.samples.append((sm, rs))
            time.sleep(0.002)
        pynvml.nvmlShutdown()

    def __enter__(self):
        self.th = threading.Thread(target=self._run, daemon=True)
        try:
            self.th.start()
            time.sleep(0.05)
        except Exception:
            self.th = None
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.th is not None:
            self.th.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"], "samples": 0}
        sm = [s for s, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workloads


class Workload:
    unit = "tokens/s"
    metric = "MoE-layer tokens/s"
    bound = "hbm"
    dtype = ("bf16 x bf16 (STQ1_0 patterns x activations) and e2m1 x e4m3 (MXFP4 x MXFP8) "
             "tensor-core products, fp32 accumulate")

    def tokens_per_step(self):
        return self.T

    def h2d_d2h(self):
        return self.T * H * 2, self.T * H * 2


class StqMatvec(Workload):
    """One STQ1_0 matrix 2048 x 6144 times one BF16 N(0,1) vector, FP32 out."""

    name = "stq_matvec"
    unit = "GB/s"
    metric = "STQ1_0 matvec achieved HBM GB/s (2048x6144, 1 token)"

    def __init__(self, S, dev):
        self.S, self.dev, self.T = S, dev, 1
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.ncopies = max(8, int(4 * l2 // STQ_MAT) + 1)
        base = S.stq1_pack(W.stq_grid_weights(I, H, dev, 0, "mv"))
        self.Wt = [base.clone() for _ in range(self.ncopies)]
        self.x = [W.bf16_normal((1, H), 1.0, dev, 0, "mvx", b) for b in range(N_BATCHES)]
        self.y = torch.empty((1, I), dtype=torch.float32, device=dev)
        self.bytes = STQ_MAT + H * 2 + I * 4

    def step(self, i, x=None, y=None):
        return self.S.stq1_gemv(self.Wt[i % self.ncopies], I, H, self.x[i % N_BATCHES] if x is None else x,
                                self.y if y is None else y)

    def accounting(self, i):
        return dict(bytes=self.bytes, flops=2 * I * H, per_kind={"gemv": dict(bytes=self.bytes)})

    def h2d_d2h(self):
        return H * 2, I * 4


class W4A8Gemm(Workload):
    """One MXFP4 expert matrix 2048 x 6144 (codes uniform, scales in [118, 127]) times
    128 BF16 N(0,1) tokens quantised on the device to MXFP8; FP32 out."""

    name = "w4a8_gemm"
    bound = "tensor"

    def __init__(self, S, dev):
        self.S, self.dev, self.T = S, dev, 128
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.ncopies = max(8, int(4 * l2 // MX_MAT) + 1)
        c, s = W.mxfp4_random(I, H, dev, 0, "w4")
        self.Wt = [(c.clone(), s.clone()) for _ in range(self.ncopies)]
        self.x = [W.bf16_normal((self.T, H), 1.0, dev, 0, "w4x", b) for b in range(N_BATCHES)]
        self.ac = torch.empty((self.T, H), dtype=torch.uint8, device=dev)
        self.asc = torch.empty((self.T, H // 32), dtype=torch.uint8, device=dev)
        self.y = torch.empty((self.T, I), dtype=torch.float32, device=dev)

    def step(self, i, x=None, y=None):
        S = self.S
        S.mxfp8_quantize_bf16(self.x[i % N_BATCHES] if x is None else x, self.ac, self.asc)
        c, s = self.Wt[i % self.ncopies]
        return S.w4a8_gemm(c, s, I, H, self.ac, self.asc, self.y if y is None else y)

    def accounting(self, i):
        fl = 2 * self.T * I * H
        by = MX_MAT + self.T * H * (1 + 1 / 32) + self.T * I * 4
        return dict(bytes=by, flops=fl, per_kind={"gemm": dict(bytes=by, flops=fl)})

    def h2d_d2h(self):
        return self.T * H * 2, self.T * I * 4


class StqPackLs(Workload):
    """The least-squares STQ1_0 encoder over one 2048 x 6144 float32 expert matrix with
    per-column importance weights exp(N(0,1)); 8 rotating matrices (400 MB > L2)."""

    name = "stq_pack_ls"
    unit = "GB/s"
    dtype = "f32 weights in, f64 decisions, u8 out"
    metric = "STQ1_0 least-squares encoder GB/s (2048x6144 float32 in, packed out)"

    def __init__(self, S, dev):
        self.S, self.dev, self.T = S, dev, 1
        self.Wf = [W.float_normal((I, H), 0.02, dev, 0, "pls", b) for b in range(N_BATCHES)]
        self.x = self.Wf   # the step's input (end-to-end timing copies it from the host)
        self.v = torch.exp(W.float_normal((H,), 1.0, dev, 0, "plsv")).contiguous()
        self.out = torch.empty(STQ_MAT, dtype=torch.uint8, device=dev)
        self.bytes = I * H * 4 + H * 4 + STQ_MAT

    def step(self, i, x=None, y=None):
        return self.S.stq1_pack_ls(self.Wf[i % N_BATCHES] if x is None else x, self.v,
                                   out=self.out if y is None else y)

    def accounting(self, i):
        return dict(bytes=self.bytes, flops=0, per_kind={"pack_ls": dict(bytes=self.bytes)})

    def h2d_d2h(self):
        return I * H * 4, STQ_MAT


class MoeLayers(Workload):
    """MoE layers of hidden 6144, 256 experts of intermediate 2048, top-8."""

    def __init__(self, S, dev, name, T, fmts, router, shared, residual, experts=E, shared_fmt="bf16"):
        global E
        E = experts
        self.S, self.dev, self.name, self.T = S, dev, name, T
        self.fmts, self.router, self.shared, self.residual = fmts, router, shared, residual
        self.shared_fmt = shared_fmt
        self.layers = [self._layer(l, f) for l, f in enumerate(fmts)]
        self.x = [W.bf16_normal((T, H), 1.0, dev, 0, name, "x", b) for b in range(N_BATCHES)]
        if not router:
            self.routing = [W.zipf_routing(T, E, K_TOP, dev, 0, name, "zipf", b) for b in range(N_BATCHES)]
        self.desc = S.make_desc(T, H, I, E, K_TOP, out_fp32=False, add_residual=residual)
        # the timed step: the RMS normalisation after the residual fused into the combine (the
        # same bits as stq_rmsnorm_bf16 on self.desc's output)
        self.step_desc = S.make_desc(T, H, I, E, K_TOP, out_fp32=False, add_residual=residual,
                                     norm_eps=W.STACK_RMS_EPS if residual else None)
        self.ws = torch.zeros(S.moe_workspace_bytes(self.desc), dtype=torch.uint8, device=dev)
        self.bufs = [torch.empty((T, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.logits = S.router_scratch(T, H, E, dev)
        self.ids = torch.empty((T, K_TOP), dtype=torch.int32, device=dev)
        self.tw = torch.empty((T, K_TOP), dtype=torch.float32, device=dev)
        self._acct = {}

    def _stq(self, l, which, rows, cols):
        S = self.S
        per = rows * cols // 256 * 42
        out = torch.empty(E * per, dtype=torch.uint8, device=self.dev)
        for e0 in range(0, E, 16):
            wf = W.stq_grid_weights(16 * rows, cols, self.dev, 0, self.name, l, which, e0)
            S.stq1_pack(wf, out=out[e0 * per:(e0 + 16) * per])
            del wf
        return out

    def _layer(self, l, fmt):
        S = self.S
        if fmt == "stq":
            mats = [self._stq(l, "g", I, H), self._stq(l, "u", I, H), self._stq(l, "d", H, I)]
            scales = [None, None, None]
        else:
            g = W.mxfp4_random(E * I, H, self.dev, 0, self.name, l, "g")
            u = W.mxfp4_random(E * I, H, self.dev, 0, self.name, l, "u")
            d = W.mxfp4_random(E * H, I, self.dev, 0, self.name, l, "d")
            mats, scales = [g[0], u[0], d[0]], [g[1], u[1], d[1]]
        sh = [None, None, None]
        if self.shared:
            sh = [W.bf16_normal((I, H), 0.02, self.dev, 0, self.name, l, "sg"),
                  W.bf16_normal((I, H), 0.02, self.dev, 0, self.name, l, "su"),
                  W.bf16_normal((H, I), 0.02, self.dev, 0, self.name, l, "sd")]
        wr = W.bf16_normal((E, H), 0.02, self.dev, 0, self.name, l, "router") if self.router else None
        f = S.FMT_STQ1_0 if fmt == "stq" else S.FMT_MXFP4
        if self.shared and self.shared_fmt == "mx8":
            q = [S.mxfp8_quantize_bf16(m) for m in sh]
            return dict(fmt=fmt, wr=wr, sh_bf16=sh,
                        w=S.ExpertWeights(f, *mats, *scales, *(c for c, _ in q), sh_fmt=S.SHARED_MXFP8,
                                          sh_gate_sc=q[0][1], sh_up_sc=q[1][1], sh_down_sc=q[2][1]))
        return dict(fmt=fmt, wr=wr, sh_bf16=sh, w=S.ExpertWeights(f, *mats, *scales, *sh))

    def step(self, i, x=None, y=None):
        S = self.S
        cur = self.x[i % N_BATCHES] if x is None else x
        for l, L in enumerate(self.layers):
            out = y if (y is not None and l == len(self.layers) - 1) else self.bufs[l % 2]
            if self.router:
                S.moe_router_topk(cur, L["wr"], K_TOP, self.logits, self.ids, self.tw)
                ids, tw = self.ids, self.tw
            else:
                ids, tw = self.routing[i % N_BATCHES]
            S.moe_expert_forward(self.step_desc, cur, ids, tw, L["w"], out, self.ws)
            cur = out
        return cur

    def touched(self, i):
        """Realised touched experts per layer for batch i (host bookkeeping, eager)."""
        S = self.S
        cur = self.x[i % N_BATCHES]
        out = []
        for l, L in enumerate(self.layers):
            if self.router:
                S.moe_router_topk(cur, L["wr"], K_TOP, self.logits, self.ids, self.tw)
                ids, tw = self.ids, self.tw
            else:
                ids, tw = self.routing[i % N_BATCHES]
            out.append(int(torch.unique(ids).numel()))
            nxt = self.bufs[(l + 1) % 2]
            S.moe_expert_forward(self.step_desc, cur, ids, tw, L["w"], nxt, self.ws)
            cur = nxt
        torch.cuda.synchronize()
        return out

    def accounting(self, i):
        """Algorithmic bytes and FLOPs of step i: the touched experts' packed matrices, the
        shared expert, the router, activations in and out; per kernel kind, per launch."""
        b = i % N_BATCHES
        if b not in self._acct:
            self._acct[b] = self.touched(b)
        n = self._acct[b]
        T, P = self.T, self.T * K_TOP
        tot, kinds = 0, {}
        sh8 = self.shared and self.shared_fmt == "mx8"
        sh_mat = MX8_MAT if sh8 else BF16_MAT
        for L, t in zip(self.layers, n):
            mat = STQ_MAT if L["fmt"] == "stq" else MX_MAT
            by = t * 3 * mat + (3 * sh_mat if self.shared else 0) + (E * H * 2 if self.router else 0) + 2 * T * H * 2
            tot += by
            if sh8:
                kinds.setdefault("shared_gate_up", []).append(
                    dict(bytes=2 * MX8_MAT + T * H * (1 + 1 / 32) + T * I * (1 + 1 / 32), flops=4 * T * I * H))
                kinds.setdefault("shared_down", []).append(
                    dict(bytes=MX8_MAT + T * I * (1 + 1 / 32) + T * H * 4, flops=2 * T * I * H))
            sh_fused = self.shared and not sh8  # BF16 shared tiles inside the STQ1_0 decode kernels
            if L["fmt"] == "stq":
                gu = t * 2 * STQ_MAT + (2 * BF16_MAT if sh_fused else 0) + T * H * 2 + (P + T) * I * 2
                dn = t * STQ_MAT + (BF16_MAT if sh_fused else 0) + (P + T) * I * 2 + (P + T) * H * 4
                kinds.setdefault("gate_up", []).append(dict(bytes=gu, flops=4 * P * I * H, touched=t))
                kinds.setdefault("down", []).append(dict(bytes=dn, flops=2 * P * I * H, touched=t))
                # prefill regime (tensor-core GEMM on MXFP8 activations): weights once, x and
                # h as MXFP8 codes + scales
                gu = t * 2 * STQ_MAT + P * H * (1 + 1 / 32) + P * I * (1 + 1 / 32)
                dn = t * STQ_MAT + P * I * (1 + 1 / 32) + P * H * 4
                kinds.setdefault("gate_up_stq_tc", []).append(dict(bytes=gu, flops=4 * P * I * H, touched=t))
                kinds.setdefault("down_stq_tc", []).append(dict(bytes=dn, flops=2 * P * I * H, touched=t))
            else:
                gu = t * 2 * MX_MAT + P * H * (1 + 1 / 32) + P * I * (1 + 1 / 32)
                dn = t * MX_MAT + P * I * (1 + 1 / 32) + P * H * 4
                kinds.setdefault("gate_up_mx", []).append(dict(bytes=gu, flops=4 * P * I * H, touched=t))
                kinds.setdefault("down_mx", []).append(dict(bytes=dn, flops=2 * P * I * H, touched=t))
        flops = len(self.layers) * 3 * 2 * T * K_TOP * I * H
        return dict(bytes=tot, flops=flops, per_kind={k: dict(bytes=float(np.mean([d["bytes"] for d in v])),
                                                             flops=float(np.mean([d.get("flops", 0) for d in v])),
                                                             touched=float(np.mean([d.get("touched", 0) for d in v])))
                                                      for k, v in kinds.items()})


class StreamLayer(MoeLayers):
    """One STQ1_0 decode layer (8 tokens, BF16 shared expert) whose routed experts sit in
    pinned host memory and stream on demand into a bank of 96 HBM slots: each step maps its
    routed ids to slots (least recently used replacement), copies the missing experts in and
    runs the layer with E = 96 on the slot ids.  Host memory stands in for the SSD sidecar of
    the 96-slot run ("Hy4-preview-FlashMoE-STQ1_0").  Routing is Zipf with one popularity
    order for every step, so consecutive steps reuse experts.  The per-step host work (slot
    mapping, copy list) cannot live in a CUDA graph: steps run eagerly."""

    N_SLOTS = 96
    POOL = 64  # routing batches, cycled

    def __init__(self, S, dev, experts=E):
        global E
        E = experts
        self.S, self.dev, self.name, self.T = S, dev, "decode_stq_stream", 8
        self.fmts, self.router, self.shared, self.residual, self.shared_fmt = ("stq",), False, True, False, "bf16"
        self.n_slots = min(self.N_SLOTS, E)
        self.host, self.slots = [], []
        for which, rows, cols in (("g", I, H), ("u", I, H), ("d", H, I)):
            per = rows * cols // 256 * 42
            host = torch.empty((E, per), dtype=torch.uint8).pin_memory()
            for e0 in range(0, E, 16):
                # same weights as the resident layer's experts (tags of MoeLayers._stq)
                wf = W.stq_grid_weights(16 * rows, cols, dev, 0, self.name, 0, which, e0)
                n = min(16, E - e0)
                host[e0:e0 + n].copy_(S.stq1_pack(wf).view(16, per)[:n])
                del wf
            self.host.append(host)
            self.slots.append(torch.zeros((self.n_slots, per), dtype=torch.uint8, device=dev))
        sh = [W.bf16_normal((I, H), 0.02, dev, 0, self.name, 0, "sg"),
              W.bf16_normal((I, H), 0.02, dev, 0, self.name, 0, "su"),
              W.bf16_normal((H, I), 0.02, dev, 0, self.name, 0, "sd")]
        self.layers = [dict(fmt="stq", wr=None, sh_bf16=sh,
                            w=S.ExpertWeights(S.FMT_STQ1_0, *(m.view(-1) for m in self.slots), None, None, None,
                                              *sh))]
        self.x = [W.bf16_normal((self.T, H), 1.0, dev, 0, self.name, "x", b) for b in range(N_BATCHES)]
        ids, tw = W.zipf_routing(self.POOL * self.T, E, K_TOP, "cpu", 0, self.name, "zipf")
        self.ids_host = [ids[b * self.T:(b + 1) * self.T].numpy().copy() for b in range(self.POOL)]
        self.tw = [tw[b * self.T:(b + 1) * self.T].to(dev) for b in range(self.POOL)]
        self.desc = S.make_desc(self.T, H, I, self.n_slots, K_TOP, out_fp32=False, regime=S.REGIME_DECODE)
        self.ws = torch.zeros(S.moe_workspace_bytes(self.desc), dtype=torch.uint8, device=dev)
        self.bufs = [torch.empty((self.T, H), dtype=torch.bfloat16, device=dev)]
        self.sid = torch.empty((self.T, K_TOP), dtype=torch.int32, device=dev)
        self.bank = S.SlotBank(E, self.n_slots)
        self.log = []           # (step, experts loaded, distinct experts) per step
        self.copy_events = None  # list of (start, stop) CUDA events around each step's copies

    def step(self, i, x=None, y=None):
        S = self.S
        b = i % self.POOL
        ids = self.ids_host[b]
        slot_ids, le, ls = self.bank.map(ids)
        if self.copy_events is not None:
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record()
        self.bank.copy(le, ls, self.host, self.slots)
        if self.copy_events is not None:
            ev[1].record()
            self.copy_events.append(ev)
        # pageable source: the runtime has read it when the call returns
        self.sid.copy_(torch.from_numpy(slot_ids), non_blocking=True)
        self.log.append((i, int(le.size), int(np.unique(ids).size)))
        cur = self.x[i % N_BATCHES] if x is None else x
        out = self.bufs[0] if y is None else y
        S.moe_expert_forward(self.desc, cur, self.sid, self.tw[b], self.layers[0]["w"], out, self.ws)
        return out

    def accounting(self, i):
        raise NotImplementedError("streamed steps are accounted from their own log")


def make_workload(name, S, dev, experts=256):
    if name == "stq_matvec":
        return StqMatvec(S, dev)
    if name == "w4a8_gemm":
        return W4A8Gemm(S, dev)
    if name == "stq_pack_ls":
        return StqPackLs(S, dev)
    if name == "decode_stq_stream":
        return StreamLayer(S, dev, experts)
    if name == "decode_mx":
        # one MXFP4 layer of the stacked workload (a small case for profiler captures)
        return MoeLayers(S, dev, name, 32, ("mx",), True, True, True, experts)
    wl = W.WORKLOADS[name]
    return MoeLayers(S, dev, name, wl.tokens, wl.formats, wl.router, wl.shared, wl.residual, experts, wl.shared_fmt)


WORKLOAD_NAMES = ["stq_matvec", "w4a8_gemm", "decode_stq", "decode_stq_sh8", "prefill_w4a8", "prefill_stq",
                  "stacked_decode", "decode_mx", "stq_pack_ls", "decode_stq_stream"]


# ----------------------------------------------------------------------------- measurement


def capture(wl):
    graphs = []
    for b in range(N_BATCHES):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            wl.step(b)
        graphs.append(g)
    return graphs


def timed_replays(graphs, steps, warmup, dist):
    for i in range(warmup):
        graphs[i % N_BATCHES].replay()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        graphs[(warmup + i) % N_BATCHES].replay()
    stop.record()
    torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    return start.elapsed_time(stop)


def kernel_times(S, wl, steps, warmup):
    """Per-kernel CUDA-event durations from graph replays (events recorded by the
    library on the launching stream, captured as event nodes)."""
    timer = S.KernelTimer(capacity=64 * N_BATCHES)
    tg = []
    with timer:
        for b in range(N_BATCHES):
            s0 = timer.st.count
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                wl.step(b)
            tg.append((g, s0, timer.st.count))
    per_kind = {}
    for i in range(steps):
        g, s0, s1 = tg[(warmup + i) % N_BATCHES]
        g.replay()
        torch.cuda.synchronize()
        for n in range(s0, s1):
            kind = S.KERNEL_KINDS[timer._kinds[n]]
            per_kind.setdefault(kind, []).append(timer.ev[2 * n].elapsed_time(timer.ev[2 * n + 1]))
    return per_kind


def e2e_steps(wl, steps, warmup):
    """Same metric end to end through the public API with pinned host buffers: H2D
    of the step's input tokens and D2H of its output inside the timed region."""
    hx = [wl.x[b].cpu().pin_memory() for b in range(N_BATCHES)]
    xs = torch.empty_like(wl.x[0])
    out = wl.step(0)
    y_dev = torch.empty_like(out)
    hy = torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory()
    for i in range(warmup):
        xs.copy_(hx[i % N_BATCHES], non_blocking=True)
        wl.step(i, x=xs, y=y_dev)
        hy.copy_(y_dev, non_blocking=True)
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(steps):
        xs.copy_(hx[(warmup + i) % N_BATCHES], non_blocking=True)
        wl.step(warmup + i, x=xs, y=y_dev)
        hy.copy_(y_dev, non_blocking=True)
    stop.record()
    torch.cuda.synchronize()
    return start.elapsed_time(stop), xs.numel() * xs.element_size(), hy.numel() * hy.element_size()


def max_over_ranks(values, device, dist):
    """Element-wise maximum of per-rank timings over all ranks (every rank calls this in
    the same order); identity on one process."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(n_ranks, units_per_rank_step, ms_per_step):
    """Units per second of the whole job: every rank processes its own units per step."""
    return n_ranks * units_per_rank_step / (ms_per_step * 1e-3)


def base_config(name, n):
    """The workload's configuration: the same dict in both arms (no measured values)."""
    return {"workload": name, "experts": E, "tokens_per_step": tokens_of(name),
            "l2": "inputs larger than L2: per-step weights exceed L2, batches rotate over 8",
            "parallelism": f"replicas x{n}"}


def run_stream(args, wl, S, dev, dist, n, rank, local):
    """The streamed layer, timed eagerly: each step (slot mapping on the host, expert copies,
    the layer) between CUDA events on the launching stream.  A second pass times every kernel
    and each step's copies; a third runs end to end with x from and y to pinned host memory.
    The host link's reference is one plain copy, measured in the same run, of one matrix of
    every expert from pinned host memory to HBM."""
    for i in range(args.warmup):
        wl.step(i)
    torch.cuda.synchronize()
    ref = torch.empty(wl.host[0].shape, dtype=torch.uint8, device=dev)
    ref.copy_(wl.host[0], non_blocking=True)
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    r0.record()
    ref.copy_(wl.host[0], non_blocking=True)
    r1.record()
    torch.cuda.synchronize()
    link_gbs = wl.host[0].numel() / (r0.elapsed_time(r1) * 1e-3) / 1e9
    del ref
    # timed pass
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wl.log = []
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        start.record()
        for i in range(args.steps):
            wl.step(args.warmup + i)
        stop.record()
        torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    clocks = clk.summary()
    ms_step = max_over_ranks([start.elapsed_time(stop)], dev, dist)[0] / args.steps
    log = list(wl.log)
    # kernel and copy times (a separate pass: the events add work)
    timer = S.KernelTimer(capacity=16 * args.steps)
    wl.copy_events, wl.log = [], []
    with timer:
        for i in range(args.steps):
            wl.step(args.warmup + args.steps + i)
    res = timer.results()
    copy_ms = [a.elapsed_time(b) for a, b in wl.copy_events]
    copied = sum(l for _, l, _ in wl.log) * 3 * STQ_MAT
    wl.copy_events = None
    kt = {}
    for kind, ms in res:
        kt.setdefault(kind, []).append(ms)
    # end to end: x in from pinned host memory, y out to it, every step
    hx = [wl.x[b].cpu().pin_memory() for b in range(N_BATCHES)]
    xs = torch.empty_like(wl.x[0])
    y_dev = torch.empty_like(wl.bufs[0])
    hy = torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory()
    torch.cuda.synchronize()
    base = args.warmup + 2 * args.steps
    wl.log = []
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for i in range(args.steps):
        xs.copy_(hx[(base + i) % N_BATCHES], non_blocking=True)
        wl.step(base + i, x=xs, y=y_dev)
        hy.copy_(y_dev, non_blocking=True)
    s1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks([s0.elapsed_time(s1)], dev, dist)[0]
    e2e_loads = float(np.mean([l for _, l, _ in wl.log]))  # the e2e pass's own misses
    loads = float(np.mean([l for _, l, _ in log]))
    distinct = float(np.mean([d for _, _, d in log]))
    copy_gbs = copied / (sum(copy_ms) * 1e-3) / 1e9 if copied else None
    out = {
        "metric": wl.metric, "value": whole_job_rate(n, wl.T, ms_step), "unit": wl.unit, "n_gpus": n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded generators; random weights on the STQ1_0 grid; Zipf routing)",
        "config": base_config(wl.name, n),
        "stream": {"slots": wl.n_slots, "experts_loaded_per_step": loads,
                   "distinct_experts_per_step": distinct, "h2d_weight_bytes_per_step": loads * 3 * STQ_MAT,
                   "l2": "inputs larger than L2: the bank (96 slots x 6.2 MB) and the copied experts"},
        "timing": "eager steps (host slot mapping, expert copies, the layer), CUDA events",
        "roofline": {"bound": "h2d", "kernel": "expert copies (cudaMemcpyAsync, pinned host to HBM)",
                     "achieved": copy_gbs, "peak": link_gbs, "unit": "GB/s",
                     "frac": copy_gbs / link_gbs if copy_gbs else None,
                     "peak_source": f"one plain pinned-host to HBM copy of {wl.host[0].numel() / 1e6:.0f} MB, "
                                    "measured in this run",
                     "traffic": None, "copy_ms_per_step": float(np.mean(copy_ms))},
        "kernels_ms": {k: statistics.mean(v) for k, v in kt.items()},
        "gpu_launches": len(res),
        "e2e": {"value": whole_job_rate(n, wl.T, e2e_ms / args.steps), "unit": wl.unit,
                "h2d_bytes_per_step": xs.numel() * xs.element_size() + wl.sid.numel() * 4 + e2e_loads * 3 * STQ_MAT,
                "d2h_bytes_per_step": hy.numel() * hy.element_size()},
        "clocks": clocks,
    }
    if rank == 0 and not dist and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(wl.name)
    if rank == 0:
        print(json.dumps(out))
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def measure(wl, S, dev, dist, n, local, steps, warmup):
    """Time one workload: CUDA graph replays of whole steps (max over ranks), per-kernel
    CUDA events, the end-to-end pass, clocks and the dominant kernel's roofline."""
    for i in range(warmup):          # eager warm-up (one-time attribute setup)
        wl.step(i)
    torch.cuda.synchronize()
    graphs = capture(wl)
    with ClockSampler(local) as clk:
        ms = timed_replays(graphs, steps, warmup, dist)
    clocks = clk.summary()
    del graphs
    ms_step = max_over_ranks([ms], dev, dist)[0] / steps
    kt = kernel_times(S, wl, steps, warmup)
    e2e_ms, h2d, d2h = e2e_steps(wl, steps, warmup)
    e2e_ms = max_over_ranks([e2e_ms], dev, dist)[0]
    acct = [wl.accounting(warmup + i) for i in range(min(steps, N_BATCHES))]
    ab = float(np.mean([a["bytes"] for a in acct]))
    pk = peaks()
    tot = {k: sum(v) for k, v in kt.items()}
    dom = max(tot, key=tot.get)
    avg_ms = tot[dom] / len(kt[dom])
    per = acct[0]["per_kind"].get(dom, {})
    launch_bytes = float(np.mean([a["per_kind"][dom]["bytes"] for a in acct if dom in a["per_kind"]])) if per else None
    launch_flops = float(np.mean([a["per_kind"][dom].get("flops", 0) for a in acct if dom in a["per_kind"]])) if per else 0
    if wl.bound == "tensor" or (dom in ("gate_up_mx", "down_mx") and wl.name == "prefill_w4a8") or \
            dom in ("gate_up_stq_tc", "down_stq_tc"):
        peak = pk["bf16"] * NOMINAL_FP8_OVER_BF16
        achieved = launch_flops / (avg_ms * 1e-3) / 1e12 if launch_flops else None
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak if achieved else None,
                "peak_source": f"{pk['src']} bf16 burst x {NOMINAL_FP8_OVER_BF16} (nominal FP8/BF16 dense ratio)",
                "frac_of_mma_microbenchmark": achieved / MMA_MICROBENCH_TFLOPS if achieved else None,
                "traffic": None, "flops_per_launch": launch_flops, "avg_launch_ms": avg_ms,
                "hbm_gbs": launch_bytes / (avg_ms * 1e-3) / 1e9 if launch_bytes else None}
    else:
        achieved = launch_bytes / (avg_ms * 1e-3) / 1e9 if launch_bytes else None
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"] if achieved else None, "peak_source": pk["src"] + " copy bandwidth",
                "traffic": None, "bytes_per_launch": launch_bytes, "avg_launch_ms": avg_ms}
    if dom in MEASURED_TRAFFIC_PER_EXPERT and wl.name not in ("prefill_w4a8", "prefill_stq") and per.get("touched"):
        touched = float(np.mean([a["per_kind"][dom]["touched"] for a in acct if dom in a["per_kind"]]))
        roof["traffic"] = MEASURED_TRAFFIC_PER_EXPERT[dom] * touched
        roof["traffic_source"] = "ncu dram bytes per touched expert (smaller case) x touched experts per launch"
    if (wl.name, dom) in MEASURED_TRAFFIC_PER_LAUNCH:
        roof["traffic"] = MEASURED_TRAFFIC_PER_LAUNCH[(wl.name, dom)]
        roof["traffic_source"] = "ncu dram bytes of one full-size launch of this kernel"
    tps = wl.tokens_per_step()
    if wl.unit == "GB/s":
        value = whole_job_rate(n, ab, ms_step) / 1e9
        e2e_val = whole_job_rate(n, ab, e2e_ms / steps) / 1e9
    else:
        value = whole_job_rate(n, tps, ms_step)
        e2e_val = whole_job_rate(n, tps, e2e_ms / steps)
    return {
        "metric": wl.metric, "value": value, "unit": wl.unit, "n_gpus": n, "steps": steps,
        "warmup": warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic (seeded generators; random weights on the format grids)",
        "config": base_config(wl.name, n),
        "accounting": {"hbm_bytes_per_step": ab,
                       "touched_experts_per_layer": getattr(wl, "_acct", {}).get(warmup % N_BATCHES),
                       "tflop_per_step": acct[0]["flops"] / 1e12},
        "timing": "CUDA graph replays, CUDA events",
        "roofline": roof,
        "kernels_ms": {k: statistics.mean(v) for k, v in kt.items()},
        "gpu_launches": int(sum(len(v) for v in kt.values())),
        "e2e": {"value": e2e_val, "unit": wl.unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clocks,
    }


# The other configurations of the target, timed in the default run after the headline
# (one GPU, one process): the single STQ1_0 matvec, the single-expert W4A8 GEMM, the
# STQ1_0 decode layer, and the two prefill layers (W4A8 and STQ1_0).
CONFIG_WORKLOADS = ["stq_matvec", "w4a8_gemm", "decode_stq", "prefill_w4a8", "prefill_stq"]


def config_summary(r):
    roof = r["roofline"]
    return {"metric": r["metric"], "value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
            "steps": r["steps"], "warmup": r["warmup"],
            "roofline": {k: roof.get(k) for k in ("bound", "kernel", "achieved", "peak", "unit", "frac",
                                                  "frac_of_mma_microbenchmark", "traffic")},
            "e2e": r["e2e"]["value"], "clocks": r["clocks"], "kernels_ms": r["kernels_ms"]}


def run_ours(args):
    dist = int(os.environ.get("WORLD_SIZE", "1")) > 1
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    n = int(os.environ.get("WORLD_SIZE", "1"))
    if dist:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import bit_quantized_moe_stq1_b200 as S

    wl = make_workload(args.workload, S, dev, args.experts)
    if args.probe_step is not None:
        # one eager step for a profiler capture of its launches, then that batch's accounting
        wl.step(args.probe_step)
        torch.cuda.synchronize(dev)
        acct = wl.accounting(args.probe_step)
        print(json.dumps({"workload": args.workload, "experts": args.experts, "probe_step": args.probe_step,
                          "batch": args.probe_step % N_BATCHES,
                          "touched_experts_per_layer": getattr(wl, "_acct", {}).get(args.probe_step % N_BATCHES),
                          "hbm_bytes": acct.get("bytes")}))
        return
    if isinstance(wl, StreamLayer):
        return run_stream(args, wl, S, dev, dist, n, rank, local)
    out = measure(wl, S, dev, dist, n, local, args.steps, args.warmup)
    del wl
    torch.cuda.empty_cache()
    if not dist and args.workload == DEFAULT_WORKLOAD and args.experts == E and not args.no_configs:
        cfg = {}
        for name in CONFIG_WORKLOADS:
            w2 = make_workload(name, S, dev, args.experts)
            cfg[name] = config_summary(measure(w2, S, dev, dist, n, local, min(args.steps, 20), args.warmup))
            del w2
            torch.cuda.empty_cache()
        out["configs"] = cfg
    if rank == 0 and not dist and not args.no_cpu:
        out["cpu_baseline"] = cpu_baseline(args.workload)
    if rank == 0:
        print(json.dumps(out))
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------------------------- oracle timing (CPU)
#
# The oracle (plain float64 numpy under oracle/) timed on the host's cores, as it stands, on
# a bounded sample of the same workload.  Its inputs are drawn on the CPU by workloads/ with
# the workloads' shapes and distributions (the CPU generators give other values than the
# GPU's); nothing here imports this package or touches the GPU.

MOE_SPECS = {
    # name: (tokens, formats per layer, router, shared, shared format, residual, prefill regime)
    "decode_stq": (8, ("stq",), True, True, "bf16", False, False),
    "decode_stq_sh8": (8, ("stq",), True, True, "mx8", False, False),
    "decode_mx": (32, ("mx",), True, True, "bf16", True, False),
    "prefill_w4a8": (4096, ("mx",), False, False, "bf16", False, True),
    "prefill_stq": (4096, ("stq",), False, False, "bf16", False, True),
    "stacked_decode": (32, ("stq", "mx") * 4, True, True, "bf16", True, False),
    "decode_stq_stream": (8, ("stq",), False, True, "bf16", False, False),
}
SINGLE_TOKENS = {"stq_matvec": 1, "w4a8_gemm": 128, "stq_pack_ls": 1}
# bytes per step of the workloads whose metric is GB/s (their algorithmic bytes)
SINGLE_BYTES = {"stq_matvec": STQ_MAT + H * 2 + I * 4, "stq_pack_ls": I * H * 4 + H * 4 + STQ_MAT}
ORACLE_POOL_MAX = 16   # packed experts per format drawn once and reused by every sample


def tokens_of(name):
    return MOE_SPECS[name][0] if name in MOE_SPECS else SINGLE_TOKENS[name]


def metric_unit_of(name):
    cls = {"stq_matvec": StqMatvec, "w4a8_gemm": W4A8Gemm, "stq_pack_ls": StqPackLs}.get(name, Workload)
    return cls.metric, cls.unit


def host_cores():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _cpu_bits(shape, std, *tag):
    return W.bf16_normal(shape, std, "cpu", 0, *tag).view(torch.int16).numpy().view(np.uint16)


class OracleSampler:
    """Times the oracle on one bounded sample per call of step(i) and scales it to one
    step of the workload; returns (seconds per step, description).

    MoE workloads: per weight format, one layer of the step: router (or the given
    routing), grouping, the activation quantisation of the MXFP8 paths, the shared expert,
    the combine and the RMS normalisation, all in full; of the layer's n touched experts, a
    uniform sample of m (each with all its tokens, its packed matrices unpacked once) runs on
    m threads, and that time is scaled by n / m; the layer time is scaled to the step's layers
    of that format.  The m packed experts come from a pool drawn once (same distributions as
    the workload's experts); numpy's own threading is off, so each thread is one core."""

    def __init__(self, name, cores=None):
        from oracle import formats as F
        from oracle import moe as M

        self.F, self.M = F, M
        self.name = name
        self.cores = cores or host_cores()
        self.pool = {}
        if name in MOE_SPECS:
            T, fmts, router, shared, sh_fmt, residual, prefill = MOE_SPECS[name]
            self.m = max(1, min(self.cores, ORACLE_POOL_MAX))
            for f in sorted(set(fmts)):
                self.pool[f] = self._threads(lambda j, f=f: self._packed_expert(f, j), range(self.m))
            self.wr = {f: _cpu_bits((E, H), 0.02, name, "oracle-router", f) for f in set(fmts)} if router else None
            if shared:
                sh = [_cpu_bits((I, H), 0.02, name, "oracle-sg"), _cpu_bits((I, H), 0.02, name, "oracle-su"),
                      _cpu_bits((H, I), 0.02, name, "oracle-sd")]
                if sh_fmt == "mx8":
                    # stored MXFP8 codes and scales, quantised once (as the GPU path's weights are)
                    sh = [F.mxfp8_quantize(F.bf16_decode(b)) for b in sh]
                self.shared = sh
        elif name == "stq_matvec":
            self.packed = F.stq1_pack(W.stq_grid_weights(I, H, "cpu", 0, name, "oracle-w").numpy())
        elif name == "w4a8_gemm":
            c, sc = W.mxfp4_random(I, H, "cpu", 0, name, "oracle-w")
            self.codes, self.scales = c.numpy(), sc.numpy()
        elif name == "stq_pack_ls":
            self.rows = 128
            self.v = torch.exp(W.float_normal((H,), 1.0, "cpu", 0, name, "oracle-v")).numpy()

    def _threads(self, fn, items):
        import concurrent.futures

        from threadpoolctl import threadpool_limits

        items = list(items)
        with threadpool_limits(limits=1):
            with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(self.cores, len(items)))) as ex:
                return list(ex.map(fn, items))

    def _packed_expert(self, fmt, j):
        F = self.F
        if fmt == "stq":
            return [F.stq1_pack(W.stq_grid_weights(r, c, "cpu", 0, self.name, "oracle-pool", which, j).numpy())
                    for which, r, c in (("g", I, H), ("u", I, H), ("d", H, I))]
        return [tuple(t.numpy() for t in W.mxfp4_random(r, c, "cpu", 0, self.name, "oracle-pool", which, j))
                for which, r, c in (("g", I, H), ("u", I, H), ("d", H, I))]

    def _expert(self, fmt, j, X, A):
        """One routed expert on its tokens: unpack its three matrices, gate/up, SwiGLU, h,
        down (float64)."""
        F, M = self.F, self.M
        shapes = ((I, H), (I, H), (H, I))
        if fmt == "stq":
            mats = [F.stq1_unpack(p_, r, c) for p_, (r, c) in zip(self.pool[fmt][j], shapes)]
        else:
            mats = [F.mxfp4_unpack(c_, s_, r, c) for (c_, s_), (r, c) in zip(self.pool[fmt][j], shapes)]
        if A is not None:
            return M.expert_ffn_mx(mats[0], mats[1], mats[2], A)["y"]
        return M.expert_ffn_bf16h(mats[0], mats[1], mats[2], X)["y"]

    def step(self, i):
        F, M = self.F, self.M
        b = i % N_BATCHES
        if self.name == "stq_matvec":
            x = _cpu_bits((1, H), 1.0, self.name, "oracle-x", b)
            t0 = time.perf_counter()
            M.stq1_gemv(self.packed, I, H, x)
            return time.perf_counter() - t0, "one full 2048 x 6144 matvec (unpack, float64 product), 1 core"
        if self.name == "w4a8_gemm":
            x = _cpu_bits((128, H), 1.0, self.name, "oracle-x", b)
            with __import__("threadpoolctl").threadpool_limits(limits=self.cores):
                t0 = time.perf_counter()
                ac, asc = F.mxfp8_quantize(F.bf16_decode(x))
                M.w4a8_gemm(self.codes, self.scales, ac, asc, I, H)
                dt = time.perf_counter() - t0
            return dt, f"the full GEMM: 128 tokens quantised, weights unpacked, float64 product ({self.cores} cores)"
        if self.name == "stq_pack_ls":
            wf = W.float_normal((self.rows, H), 0.02, "cpu", 0, self.name, "oracle-w", b).numpy()
            t0 = time.perf_counter()
            F.stq1_pack_ls(wf, self.v)
            return (time.perf_counter() - t0) * (I / self.rows), f"{self.rows} of the {I} rows, scaled to the matrix"
        T, fmts, router, shared, sh_fmt, residual, prefill = MOE_SPECS[self.name]
        P = T * K_TOP
        total, desc = 0.0, []
        rng = np.random.default_rng(i)
        for f in sorted(set(fmts)):
            nl = sum(1 for g in fmts if g == f)
            xb = _cpu_bits((T, H), 1.0, self.name, "oracle-x", f, b)
            if not router:
                ids_t, tw_t = W.zipf_routing(T, E, K_TOP, "cpu", 0, self.name, "oracle-zipf", b)
                ids, tw = ids_t.numpy(), tw_t.double().numpy()
            t0 = time.perf_counter()
            if router:
                ids, tw, _ = M.router_topk(xb, self.wr[f], K_TOP)
            counts, offsets, perm, inv = M.permute(ids, E)
            X = F.bf16_decode(xb)
            A = None
            if f == "mx" or prefill:
                qc, qs = F.mxfp8_quantize(X)
                A = F.mxfp8_dequantize(qc, qs)
            y_sh = 0.0
            if shared and sh_fmt == "mx8":
                sh = [F.mxfp8_dequantize(c_, s_) for c_, s_ in self.shared]
                qc, qs = F.mxfp8_quantize(X)
                y_sh = M.expert_ffn_mx(sh[0], sh[1], sh[2], F.mxfp8_dequantize(qc, qs))["y"]
            elif shared:
                sh = [F.bf16_decode(m_) for m_ in self.shared]
                y_sh = M.expert_ffn_bf16h(sh[0], sh[1], sh[2], X)["y"]
            t_fixed = time.perf_counter() - t0
            touched = np.flatnonzero(counts)
            pick = np.sort(rng.choice(touched, size=min(self.m, touched.size), replace=False))
            jobs = [(j, perm[offsets[e]:offsets[e + 1]] // K_TOP) for j, e in enumerate(pick)]
            t0 = time.perf_counter()
            ys = self._threads(lambda jt: self._expert(f, jt[0], X[jt[1]], None if A is None else A[jt[1]]), jobs)
            t_exp = time.perf_counter() - t0
            # combine (all pairs; the sampled experts' outputs stand in for the rest) and norm
            Yp = np.zeros((P, H))     # sorted pair order
            for (j, toks), ye in zip(jobs, ys):
                Yp[offsets[pick[j]]:offsets[pick[j]] + len(toks)] = ye
            t0 = time.perf_counter()
            y, _ = M.combine(Yp[inv], np.abs(Yp[inv]), tw, y_sh if shared else None, None, X if residual else None)
            if residual:
                M.rms_norm(y, W.STACK_RMS_EPS)
            t_fixed += time.perf_counter() - t0
            per_layer = t_fixed + t_exp * touched.size / pick.size
            total += nl * per_layer
            desc.append(f"{f}: {nl} layer(s) x ({t_fixed:.2f} s router/grouping/quant/shared/combine/norm in full + "
                        f"{t_exp:.2f} s for {pick.size} of {touched.size} touched experts on {pick.size} threads, "
                        f"x {touched.size / pick.size:.1f})")
        return total, "; ".join(desc)

    def threads_used(self):
        if self.name in MOE_SPECS:
            return self.m
        return self.cores if self.name == "w4a8_gemm" else 1


def cpu_baseline(name, budget_s=12.0, sampler=None):
    """The oracle on a bounded sample of the workload, scaled to the metric's unit."""
    smp = sampler or OracleSampler(name)
    times, t0, desc = [], time.perf_counter(), ""
    while True:
        dt, desc = smp.step(len(times))
        times.append(dt)
        if time.perf_counter() - t0 > budget_s or len(times) >= 20 or name in MOE_SPECS:
            break
    dt = statistics.mean(times)
    _, unit = metric_unit_of(name)
    value = SINGLE_BYTES[name] / dt / 1e9 if unit == "GB/s" else tokens_of(name) / dt
    return {"value": value, "unit": unit, "cores": smp.threads_used(), "kind": "oracle",
            "sample": f"{desc}; {len(times)} sample(s), mean {dt:.2f} s per step"}


def run_reference(args):
    """The oracle arm: rank 0 alone times the CPU oracle, one bounded sample per step; the
    other ranks exit without work.  Never imports this package and never touches a GPU."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload
    smp = OracleSampler(name)
    metric, unit = metric_unit_of(name)
    secs, desc = [], ""
    for i in range(args.warmup + args.steps):
        dt, desc = smp.step(i)
        if i >= args.warmup:
            secs.append(dt)
    ms = 1e3 * statistics.mean(secs)
    value = SINGLE_BYTES[name] / (ms * 1e-3) / 1e9 if unit == "GB/s" else tokens_of(name) / (ms * 1e-3)
    out = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": base_config(name, args.gpus),
           "cpu_baseline": {"value": value, "unit": unit, "cores": smp.threads_used(), "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_NAMES)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other configurations timed after the default workload")
    ap.add_argument("--experts", type=int, default=256,
                    help="routed experts per layer (256 = the workloads; fewer only for small profiler captures)")
    ap.add_argument("--probe-step", type=int, default=None,
                    help="run step i once, eagerly, print that batch's touched experts and exit (for counter captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
