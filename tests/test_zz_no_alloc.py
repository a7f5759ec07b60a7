"""The router entry point that allocates nothing: moe_router_topk_static keeps its
scratch in a fixed array inside the library, for callers that cannot allocate a
scratch buffer.  It must give the same experts and weights as moe_router_topk on
two calls in a row (the second call sees the first call's leftovers in the array).
Collected last on purpose; it also passes when run alone in a fresh process."""

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def S():
    import bit_quantized_moe_stq1_b200 as S
    return S


def _same_choice(ids_a, w_a, ids_b, w_b, logits):
    ids_a, ids_b = ids_a.cpu().numpy(), ids_b.cpu().numpy()
    w_a, w_b = w_a.cpu().double().numpy(), w_b.cpu().double().numpy()
    lg = logits.cpu().double().numpy()
    k = ids_a.shape[1]
    for t in range(ids_a.shape[0]):
        srt = np.sort(lg[t])[::-1]
        if srt[k - 1] - srt[k] < 1e-6 * max(1.0, abs(srt[0])):
            continue   # near-tie at the k-th place: either choice is valid
        assert set(ids_a[t]) == set(ids_b[t])
        for j, e in enumerate(ids_a[t]):
            assert abs(w_a[t, j] - w_b[t, list(ids_b[t]).index(e)]) <= 1e-5


@pytest.mark.parametrize("first,second", [((32, 6144, 256, 8), (3, 512, 20, 4)),
                                          ((8, 6144, 256, 8), (200, 6144, 256, 8))])
def test_static_router_matches_scratch_router(S, first, second):
    for call, (T, H, E, k) in enumerate((first, second)):
        x = W.bf16_normal((T, H), 1.0, DEV, 0, "noalloc-x", call, T, H)
        wr = W.bf16_normal((E, H), 0.02, DEV, 0, "noalloc-r", call, E, H)
        ids_ref, w_ref, logits = S.moe_router_topk(x, wr, k)
        ids, w = S.moe_router_topk_static(x, wr, k)
        torch.cuda.synchronize()
        _same_choice(ids_ref, w_ref, ids, w, logits)


def test_static_router_rejects_oversize(S):
    # 8 slices x 300 tokens x 256 experts > 524288 floats: refused before any launch
    x = torch.zeros((300, 6144), dtype=torch.bfloat16, device=DEV)
    wr = torch.zeros((256, 6144), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(S.StqError) as e:
        S.moe_router_topk_static(x, wr, 8)
    assert e.value.status == -7
