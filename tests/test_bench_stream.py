"""bench.py's streamed-layer workload without a GPU: the real slot bank and bookkeeping,
with the GPU-only calls (pack, layer, events, pinning, clock sampling) replaced by fakes
that check what they are given.  The layer runs on slot ids below the slot count, every
expert a step routes to is in its slot when the layer runs, and the JSON line carries the
streaming fields."""

import json

import numpy as np
import pytest
import torch


class _Event:
    def __init__(self, enable_timing=False):
        pass

    def record(self):
        pass

    def elapsed_time(self, other):
        return 1.0


class _Timer:
    def __init__(self, capacity=512):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass

    def results(self):
        return [("gate_up", 0.2), ("down", 0.1)]


class _Clock:
    def __init__(self, gpu_index):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        pass

    def summary(self):
        return {"sm_mhz": None}


def test_streamed_layer_host_path(monkeypatch, capsys):
    import bench
    import bit_quantized_moe_stq1_b200 as S

    seen = {"layers": 0, "loads": 0}

    def pack(w, out=None, err=None, stream=None):
        rows, K = w.shape
        return torch.zeros(rows * K // 256 * 42, dtype=torch.uint8)

    def copy(self, le, ls, src, dst, stream=None):
        for m in range(len(src)):
            for e, s in zip(le.tolist(), ls.tolist()):
                dst[m][s].copy_(src[m][e])
        seen["loads"] += len(le)

    def forward(desc, x, ids, tw, w, y, ws, stream=None):
        assert ids.dtype == torch.int32 and tuple(ids.shape) == (desc.T, desc.k)
        assert 0 <= int(ids.min()) and int(ids.max()) < desc.E
        assert w.gate.numel() == desc.E * desc.I * desc.H // 256 * 42
        # the slots the layer reads hold the experts the step routed to
        slot_expert = wl.bank.resident()
        routed = wl.ids_host[wl.log[-1][0] % wl.POOL]
        assert np.array_equal(slot_expert[ids.numpy()], routed)
        for m, host in zip(wl.slots, wl.host):
            for s in np.unique(ids.numpy()):
                assert torch.equal(m[s], host[slot_expert[s]])
        seen["layers"] += 1

    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(S, "stq1_pack", pack)
    monkeypatch.setattr(S, "moe_expert_forward", forward)
    monkeypatch.setattr(S.SlotBank, "copy", copy)
    monkeypatch.setattr(S, "KernelTimer", _Timer)
    monkeypatch.setattr(bench, "ClockSampler", _Clock)
    # the fake pack reads only the shape: skip drawing full-size weights
    monkeypatch.setattr(bench.W, "stq_grid_weights", lambda rows, K, *a: torch.empty(1).expand(rows, K))
    # 64 experts in 40 slots: the busiest step of this routing touches 36, and the steps
    # together touch more than 40, so the bank evicts
    monkeypatch.setattr(bench.StreamLayer, "N_SLOTS", 40)

    wl = bench.make_workload("decode_stq_stream", S, "cpu", 64)
    # distinct host bytes per expert, so a wrong copy is visible
    for h in wl.host:
        h.copy_(torch.arange(64, dtype=torch.uint8).view(64, 1).expand_as(h))

    class Args:
        workload, experts, warmup, steps, no_cpu, gpus = "decode_stq_stream", 64, 3, 6, True, 1

    bench.run_stream(Args, wl, S, "cpu", False, 1, 0, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert seen["layers"] == 3 + 3 * 6
    assert seen["loads"] > 40                       # the 40-slot bank evicted
    assert line["stream"]["slots"] == 40 and line["config"]["workload"] == "decode_stq_stream"
    assert line["roofline"]["bound"] == "h2d" and line["gpu_launches"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] >= 8 * 6144 * 2
    assert 0 < line["stream"]["experts_loaded_per_step"] <= line["stream"]["distinct_experts_per_step"] <= 40
