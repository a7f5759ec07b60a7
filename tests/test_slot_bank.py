"""Host-side expert slot bank (no GPU): the native bank against a plain statement of its
replacement rule, per-call invariants, errors that leave the bank unchanged, and the
copy call's argument checks (which return before any CUDA call)."""

import ctypes

import numpy as np
import pytest


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


class ReferenceBank:
    """The documented rule: hits keep their slot; each miss, in first-use order, takes the
    least recently used slot that the call does not need (empty slots first, ties to the
    lowest index)."""

    def __init__(self, n_experts, n_slots):
        self.slot_expert = [-1] * n_slots
        self.slot_used = [-1] * n_slots
        self.clock = 0

    def map(self, ids):
        distinct = list(dict.fromkeys(int(e) for e in ids))
        now = self.clock
        self.clock += 1
        where = {e: s for s, e in enumerate(self.slot_expert) if e >= 0}
        for e in distinct:
            if e in where:
                self.slot_used[where[e]] = now
        loads = []
        for e in distinct:
            if e in where:
                continue
            free = [s for s in range(len(self.slot_expert)) if self.slot_used[s] != now]
            victim = min(free, key=lambda s: (self.slot_used[s], s))
            if self.slot_expert[victim] >= 0:
                del where[self.slot_expert[victim]]
            self.slot_expert[victim] = e
            self.slot_used[victim] = now
            where[e] = victim
            loads.append((e, victim))
        return [where[int(e)] for e in ids], loads


@pytest.mark.parametrize("n_experts,n_slots,topk,tokens", [(256, 8, 8, 1), (256, 96, 8, 4), (64, 24, 4, 5),
                                                           (16, 16, 2, 3)])
def test_matches_the_replacement_rule(S, n_experts, n_slots, topk, tokens):
    rng = np.random.default_rng(n_experts * 1000 + n_slots)
    # Zipf-like popularity so that hits and evictions both happen
    p = 1.0 / np.arange(1, n_experts + 1) ** 1.1
    p /= p.sum()
    bank, ref = S.SlotBank(n_experts, n_slots), ReferenceBank(n_experts, n_slots)
    for _ in range(200):
        ids = np.stack([rng.choice(n_experts, size=topk, replace=False, p=p) for _ in range(tokens)]).astype(np.int32)
        if len(np.unique(ids)) > n_slots:
            continue
        slots, le, ls = bank.map(ids)
        rslots, rloads = ref.map(ids.reshape(-1))
        assert np.array_equal(slots.reshape(-1), np.array(rslots, dtype=np.int32))
        assert list(zip(le.tolist(), ls.tolist())) == rloads
        res = bank.resident()
        assert np.array_equal(res[slots], ids)                       # every id's slot holds it
        held = res[res >= 0]
        assert len(np.unique(held)) == len(held)                     # no expert in two slots
        assert len(set(le.tolist())) == len(le) and set(le.tolist()) <= set(ids.reshape(-1).tolist())


def test_repeat_is_all_hits_and_top8_fits_eight_slots(S):
    bank = S.SlotBank(256, 8)
    ids = np.array([[3, 17, 200, 5, 9, 41, 99, 128]], dtype=np.int32)
    s1, le1, _ = bank.map(ids)
    assert len(le1) == 8 and sorted(s1.reshape(-1).tolist()) == list(range(8))
    s2, le2, _ = bank.map(ids)
    assert len(le2) == 0 and np.array_equal(s1, s2)
    # empty slots fill in first-use order: expert 99 sits in slot 6 and 128 in slot 7; a call
    # that keeps six of the experts and brings two new ones evicts exactly those two slots
    assert s1.reshape(-1).tolist() == list(range(8))
    ids3 = np.array([[3, 17, 200, 5, 9, 41, 7, 8]], dtype=np.int32)
    s3, le3, ls3 = bank.map(ids3)
    assert le3.tolist() == [7, 8] and ls3.tolist() == [6, 7]
    assert s3.reshape(-1).tolist() == list(range(8))


def test_errors_leave_the_bank_unchanged(S):
    bank = S.SlotBank(32, 4)
    bank.map(np.array([1, 2, 3], dtype=np.int32))
    before = bank.resident().copy()
    with pytest.raises(S.StqError):
        bank.map(np.array([4, 5, 6, 7, 8], dtype=np.int32))          # five distinct experts, four slots
    with pytest.raises(S.StqError):
        bank.map(np.array([1, 32], dtype=np.int32))                  # id outside [0, 32)
    with pytest.raises(S.StqError):
        bank.map(np.array([-1], dtype=np.int32))
    assert np.array_equal(bank.resident(), before)
    slots, le, _ = bank.map(np.zeros(0, dtype=np.int32))             # an empty call is fine
    assert slots.size == 0 and le.size == 0


def test_create_rejects_bad_sizes(S):
    for n_e, n_s in [(0, 1), (8, 0), (8, 9), (-1, -1)]:
        with pytest.raises(S.StqError):
            S.SlotBank(n_e, n_s)


def test_copy_argument_checks_need_no_gpu(S):
    """Every case below fails an argument check, which returns before any CUDA call."""
    lib = S.lib
    bank = S.SlotBank(32, 4)
    h = bank._h
    e = (ctypes.c_int32 * 1)(0)
    s = (ctypes.c_int32 * 1)(0)
    assert lib.stq_slot_bank_copy(h, e, s, 0, 3, None, None, None, None) == 0       # nothing to copy
    assert lib.stq_slot_bank_copy(None, e, s, 1, 1, None, None, None, None) == -1   # no bank
    assert lib.stq_slot_bank_copy(h, e, s, 1, 1, None, None, None, None) == -1      # null arrays
    src = (ctypes.c_void_p * 1)(None)
    dst = (ctypes.c_void_p * 1)(None)
    sz = (ctypes.c_size_t * 1)(16)
    assert lib.stq_slot_bank_copy(h, e, s, 1, 1, src, dst, sz, None) == -1          # null matrix pointers
    src2 = (ctypes.c_void_p * 1)(1 << 20)
    dst2 = (ctypes.c_void_p * 1)(1 << 21)
    for ex, sl in ((-1, 0), (32, 0), (0, -1), (0, 4)):                              # outside 32 experts, 4 slots
        ee, ss = (ctypes.c_int32 * 1)(ex), (ctypes.c_int32 * 1)(sl)
        assert lib.stq_slot_bank_copy(h, ee, ss, 1, 1, src2, dst2, sz, None) == -1, (ex, sl)


def test_copy_binding_checks_shapes(S):
    import torch

    bank = S.SlotBank(8, 2)
    src = [torch.zeros((8, 64), dtype=torch.uint8)]
    with pytest.raises(ValueError):
        bank.copy([0], [0], src, [torch.zeros((3, 64), dtype=torch.uint8)])   # 3 rows for 2 slots
    with pytest.raises(ValueError):
        bank.copy([0], [0], src, [])                                           # one destination per matrix
    with pytest.raises(ValueError):
        bank.copy([0], [0], src, [torch.zeros((2, 64), dtype=torch.uint8)])   # destination not on the GPU
