"""The router entry point that allocates nothing: moe_router_topk_static keeps its
scratch in a fixed array inside the library, for callers that cannot allocate a
scratch buffer.  It must give the same experts and weights as moe_router_topk on
two calls in a row (the second call sees the first call's leftovers in the array),
and both must agree with the oracle's router away from near-ties at the k-th place.
Collected last on purpose; it also passes when run alone in a fresh process."""

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe as M

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT_FLOATS = 524288   # the fixed array: 2 MiB of float32 per GPU


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _same_choice(ids_a, w_a, ids_b, w_b, p):
    """Same expert set and weights within 1e-5, except where the k-th and (k+1)-th
    probabilities of p (the oracle's softmax) are within 1e-6 of each other."""
    ids_a, ids_b = np.asarray(ids_a), np.asarray(ids_b)
    w_a, w_b = np.asarray(w_a, dtype=np.float64), np.asarray(w_b, dtype=np.float64)
    k = ids_a.shape[1]
    for t in range(ids_a.shape[0]):
        ps = np.sort(p[t])[::-1]
        if k < ps.size and ps[k - 1] - ps[k] < 1e-6 * ps[0]:
            continue   # near-tie at the k-th place: either choice is valid
        assert set(ids_a[t]) == set(ids_b[t])
        for j, e in enumerate(ids_a[t]):
            assert abs(w_a[t, j] - w_b[t, list(ids_b[t]).index(e)]) <= 1e-5


def _check_against_oracle_and_scratch(S, x, wr, k):
    ids_ref, w_ref, _ = S.moe_router_topk(x, wr, k)
    ids, w = S.moe_router_topk_static(x, wr, k)
    torch.cuda.synchronize()
    ri, rw, p = M.router_topk(_bits(x), _bits(wr), k)
    ids_n, w_n = ids.cpu().numpy(), w.cpu().double().numpy()
    assert ids_n.min() >= 0 and ids_n.max() < wr.shape[0]
    _same_choice(ids_n, w_n, ri, rw, p)                                          # against the oracle
    _same_choice(ids_n, w_n, ids_ref.cpu().numpy(), w_ref.cpu().double().numpy(), p)  # against the scratch router
    assert np.allclose(w_n.sum(axis=1), 1.0, atol=1e-5)


@pytest.mark.parametrize("first,second", [((32, 6144, 256, 8), (3, 512, 20, 4)),
                                          ((8, 6144, 256, 8), (200, 6144, 256, 8)),
                                          ((5, 256, 64, 8), (17, 256, 300, 2))])
def test_static_router_matches_oracle_and_scratch_router(S, first, second):
    """Two calls in a row; H = 256 takes the one-slice path of the logits kernel."""
    for call, (T, H, E, k) in enumerate((first, second)):
        x = W.bf16_normal((T, H), 1.0, DEV, 0, "noalloc-x", call, T, H)
        wr = W.bf16_normal((E, H), 0.02, DEV, 0, "noalloc-r", call, E, H)
        _check_against_oracle_and_scratch(S, x, wr, k)


def test_static_router_at_the_size_limit(S):
    """8 slices x 256 tokens x 256 experts = exactly 524,288 floats: accepted and correct."""
    T, H, E, k = 256, 6144, 256, 8
    assert S.lib.stq_router_ksplit(H) * T * E == LIMIT_FLOATS
    x = W.bf16_normal((T, H), 1.0, DEV, 0, "noalloc-limit-x")
    wr = W.bf16_normal((E, H), 0.02, DEV, 0, "noalloc-limit-r")
    _check_against_oracle_and_scratch(S, x, wr, k)


def test_static_router_empty_batch(S):
    x = torch.zeros((0, 6144), dtype=torch.bfloat16, device=DEV)
    wr = W.bf16_normal((256, 6144), 0.02, DEV, 0, "noalloc-empty-r")
    ids, w = S.moe_router_topk_static(x, wr, 8)
    torch.cuda.synchronize()
    assert ids.shape == (0, 8) and w.shape == (0, 8)


def test_static_router_rejects_oversize(S):
    # 8 slices x 257 tokens x 256 experts is one token past 524288 floats: refused
    # before any launch, outputs untouched
    x = torch.zeros((257, 6144), dtype=torch.bfloat16, device=DEV)
    wr = torch.zeros((256, 6144), dtype=torch.bfloat16, device=DEV)
    ids = torch.full((257, 8), -7, dtype=torch.int32, device=DEV)
    with pytest.raises(S.StqError) as e:
        S.moe_router_topk_static(x, wr, 8, ids=ids)
    assert e.value.status == -7
    assert bool((ids == -7).all())
