"""Host-to-HBM expert streaming on the GPU: routed experts in pinned host memory, a slot
bank in HBM, the layer run on slot ids.  Checked stage by stage against the oracle with
the weights each slot holds, and against the layer with every expert resident.  Collected
after the other GPU tests."""

import numpy as np
import pytest
import torch

import workloads as W
from test_gpu_moe import _check_layer, _make_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def test_moe_stq_slot_bank_streaming(S):
    """Routed experts streamed from pinned host memory into an 8-slot HBM bank over six
    calls with Zipf routing (empty slots filled, hits, evictions): each call maps its ids
    to slots, copies the misses in and runs the layer on the slot ids with E = 8.  Each
    call is checked stage by stage against the oracle with the weights the bank says each
    slot holds, and against the same layer run with all 32 experts resident."""
    T, H, I, E, k, n_slots, calls = 4, 512, 256, 32, 2, 8, 6
    tag = ("slot-bank", T, H, I, E, k)
    gw, packs, sh, _, x = _make_layer(S, T, H, I, E, k, True, tag)
    gw_cpu = [m.cpu() for m in gw]
    rows = (I, I, H)
    host = [p.view(E, -1).cpu().pin_memory() for p in packs]
    bank_w = [torch.zeros((n_slots, h.shape[1]), dtype=torch.uint8, device=DEV) for h in host]
    bank = S.SlotBank(E, n_slots)
    desc_res = S.make_desc(T, H, I, E, k, out_fp32=True, regime=S.REGIME_DECODE)
    desc = S.make_desc(T, H, I, n_slots, k, out_fp32=True, regime=S.REGIME_DECODE)
    ws_res = torch.zeros(S.moe_workspace_bytes(desc_res), dtype=torch.uint8, device=DEV)
    ws = torch.zeros(S.moe_workspace_bytes(desc), dtype=torch.uint8, device=DEV)
    ew_res = S.ExpertWeights(S.FMT_STQ1_0, *packs, None, None, None, *sh)
    ew = S.ExpertWeights(S.FMT_STQ1_0, *(b.view(-1) for b in bank_w), None, None, None, *sh)
    ids_all, tw_all = W.zipf_routing(calls * T, E, k, "cpu", 0, tag, "ids")
    n_loads = 0
    for c in range(calls):
        ids = ids_all[c * T:(c + 1) * T].contiguous()
        slot_ids, le, ls = bank.map(ids.numpy())
        bank.copy(le, ls, host, bank_w)
        n_loads += le.size
        sid = torch.from_numpy(slot_ids).to(DEV)
        tw = tw_all[c * T:(c + 1) * T].contiguous().to(DEV)
        y = torch.empty((T, H), dtype=torch.float32, device=DEV)
        S.moe_expert_forward(desc, x, sid, tw, ew, y, ws)
        assert S.moe_get_device_error(ws) == 0
        y_res = torch.empty((T, H), dtype=torch.float32, device=DEV)
        S.moe_expert_forward(desc_res, x, ids.to(DEV), tw, ew_res, y_res, ws_res)
        assert S.moe_get_device_error(ws_res) == 0
        # the dense weights each slot holds now, in slot order (empty slots as zeros)
        held = bank.resident()
        gw_slots = [torch.cat([m[int(e) * R:(int(e) + 1) * R] if e >= 0 else torch.zeros_like(m[:R]) for e in held])
                    for m, R in zip(gw_cpu, rows)]
        P = T * k
        r = dict(
            gw=gw_slots, sh=sh, sh_mx8=None, x=x, ids=slot_ids, tw=tw.cpu().double().numpy(),
            y=y.cpu().double().numpy(),
            h=S.moe_workspace_view(desc, ws, "h", torch.bfloat16, (P + T, I)).float().cpu().double().numpy(),
            Y=S.moe_workspace_view(desc, ws, "Y", torch.float32, (P + T, H)).cpu().double().numpy(),
            perm=S.moe_workspace_view(desc, ws, "perm", torch.int32, (P,)).cpu().numpy(),
            inv=S.moe_workspace_view(desc, ws, "inv", torch.int32, (P,)).cpu().numpy(),
        )
        _check_layer(r, T, H, I, n_slots, k)
        # the same layer with every expert resident: a wrong or stale slot is off by O(1)
        yr = y_res.cpu().double().numpy()
        assert np.all(np.abs(r["y"] - yr) <= 1e-4 * np.abs(yr) + 1e-5), float(np.max(np.abs(r["y"] - yr)))
    assert n_loads > n_slots  # the bank evicted
