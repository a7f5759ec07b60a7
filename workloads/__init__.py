"""Seeded synthetic inputs for the routed-expert FFN workloads.

This module only draws random numbers with the shapes and distributions of the
five workloads; it holds no packing, quantisation or MoE arithmetic.  Both the
CUDA path (tests, bench) and the CPU oracle take their inputs from here.  Every
tensor is drawn from its own ``torch.Generator`` seeded from (seed, tag), on the
device the caller names, so a tensor is reproducible on that device.

Workloads (shapes from "Hy4-preview-FlashMoE-STQ1_0", "Package details":
hidden 6144, MoE intermediate 2048, 256 routed experts, top-8, 1 shared expert):

* ``stq_matvec``   one STQ1_0 matrix 2048 x 6144 times one BF16 N(0,1) vector.
* ``w4a8_gemm``    one MXFP4 expert matrix 2048 x 6144 times 128 BF16 tokens.
* ``decode_stq``   one MoE layer, STQ1_0 experts, 8 tokens, BF16 router, shared expert.
* ``prefill_w4a8`` one MoE layer, MXFP4 experts, 4096 tokens, Zipf(1.1) routing.
* ``stacked_decode`` 8 MoE layers (odd layers STQ1_0, even layers MXFP4), 32
  tokens, fresh router per layer, residual add, then an RMS normalisation
  (unit gain, eps ``STACK_RMS_EPS``) of each layer's output before the next layer.
"""

import hashlib
from dataclasses import dataclass

import torch

HIDDEN = 6144
INTER = 2048
EXPERTS = 256
TOPK = 8


@dataclass(frozen=True)
class Workload:
    name: str
    tokens: int
    layers: int
    formats: tuple          # per layer: "stq" or "mx"
    router: bool            # BF16 router (else Zipf routing)
    shared: bool            # shared BF16 expert
    residual: bool
    shared_fmt: str = "bf16"  # shared expert storage: "bf16" or "mx8" (MXFP8 W8A8 g32)
    H: int = HIDDEN
    I: int = INTER
    E: int = EXPERTS
    k: int = TOPK


WORKLOADS = {
    "stq_matvec": Workload("stq_matvec", 1, 1, ("stq",), False, False, False, E=1, k=1),
    "w4a8_gemm": Workload("w4a8_gemm", 128, 1, ("mx",), False, False, False, E=1, k=1),
    "decode_stq": Workload("decode_stq", 8, 1, ("stq",), True, True, False),
    "decode_stq_sh8": Workload("decode_stq_sh8", 8, 1, ("stq",), True, True, False, shared_fmt="mx8"),
    "prefill_w4a8": Workload("prefill_w4a8", 4096, 1, ("mx",), False, False, False),
    "prefill_stq": Workload("prefill_stq", 4096, 1, ("stq",), False, False, False),
    "stacked_decode": Workload("stacked_decode", 32, 8, ("stq", "mx") * 4, True, True, True),
}


def _seed(seed, *tag):
    h = hashlib.sha256(repr((seed,) + tuple(tag)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(device, seed, *tag):
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, *tag))
    return g


def bf16_normal(shape, std, device, seed, *tag):
    """BF16 N(0, std^2) (drawn in float32, then cast)."""
    g = generator(device, seed, *tag)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def stq_grid_weights(rows, K, device, seed, *tag):
    """Float32 weights on the 3:4 ternary grid: per group of four consecutive k,
    the zero lane uniform in 0..3 and the other lanes' signs uniform +-1; per
    256-block of a row, d = |N(0, 0.02)| cast to FP16.  w = d * {0, +-1}."""
    assert K % 256 == 0
    g = generator(device, seed, *tag)
    z = torch.randint(0, 4, (rows, K // 4, 1), generator=g, device=device)
    sgn = torch.randint(0, 2, (rows, K // 4, 4), generator=g, device=device, dtype=torch.int8)
    d = (torch.randn((rows, K // 256), generator=g, device=device) * 0.02).abs().half().float()
    lane = torch.arange(4, device=device).view(1, 1, 4)
    pat = torch.where(lane == z, 0.0, sgn.float() * 2.0 - 1.0)
    return (pat.view(rows, K // 256, 256) * d.unsqueeze(-1)).view(rows, K).contiguous()


def mxfp4_random(rows, K, device, seed, *tag, emin=118, emax=127):
    """MXFP4 weights as stored: codes uniform over the 16 E2M1 codes (uniform
    bytes, two codes per byte) and one UE8M0 exponent per 32 along K uniform in
    [emin, emax] (the single-expert and prefill workloads use [118, 127])."""
    g = generator(device, seed, *tag)
    codes = torch.randint(0, 256, (rows, K // 2), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    scales = torch.randint(emin, emax + 1, (rows, K // 32), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    return codes, scales


# Stacked decode: eps of the RMS normalisation between layers.
STACK_RMS_EPS = 1e-6


def float_normal(shape, std, device, seed, *tag):
    g = generator(device, seed, *tag)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def zipf_routing(T, E, k, device, seed, *tag, s=1.1):
    """Per token k distinct experts drawn one after another without replacement
    with probability proportional to (rank + 1)^-s, ranks over a seeded random
    permutation of the E experts; weights Dirichlet(1) over the k (normalised
    Exp(1) draws).  Returns (ids [T, k] int32, w [T, k] float32)."""
    g = generator(device, seed, *tag)
    perm = torch.randperm(E, generator=g, device=device)
    pop = torch.empty(E, device=device, dtype=torch.float64)
    pop[perm] = (torch.arange(E, device=device, dtype=torch.float64) + 1.0) ** (-s)
    ids = torch.multinomial(pop.expand(T, E), k, replacement=False, generator=g).to(torch.int32)
    ex = -torch.log(torch.rand((T, k), generator=g, device=device, dtype=torch.float64).clamp_min(1e-300))
    w = (ex / ex.sum(dim=1, keepdim=True)).to(torch.float32)
    return ids.contiguous(), w.contiguous()


def uniform_routing(T, E, k, device, seed, *tag):
    """k distinct experts per token, uniform; weights Dirichlet(1)."""
    g = generator(device, seed, *tag)
    ids = torch.stack([torch.randperm(E, generator=g, device=device)[:k] for _ in range(T)]).to(torch.int32)
    ex = -torch.log(torch.rand((T, k), generator=g, device=device, dtype=torch.float64).clamp_min(1e-300))
    return ids.contiguous(), (ex / ex.sum(dim=1, keepdim=True)).to(torch.float32).contiguous()
