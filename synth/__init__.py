"""Seeded synthetic inputs for the decode GEMM, shared by the tests, the
benchmark and the oracle checks.

This module holds workload definitions and random-number draws only: none of
the GEMM's arithmetic.  Recipe (one reading of the workloads, since the pages
print no data):

* X ~ N(0, 1) and W ~ N(0, 1/K) (standard deviation 1/sqrt(K)), drawn in fp32
  and rounded to bf16 by torch (round to nearest even).
* One CPU ``torch.Generator`` seeded with ``seed`` draws X first, then W.
* Chain task t uses seed t for its X and seed 10000 + t for its W.

Shapes are those of the decode linears of a Qwen3-8B-sized dense model
(d = 4096, d_ff = 12288, GQA 32 query / 8 key-value heads of 128: fused QKV
4096 -> 6144, o 4096 -> 4096, fused gate_up 4096 -> 24576, down 12288 -> 4096;
"Fleet ..." reading notes, Summary and section 1), and of the skinny
production shapes the FlyDSL article benchmarks (K = 7168 and 8192; the
article prints no list, so these stand in for it).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# (name, K, N) of one decoder layer's linears, Qwen3-8B-sized.
QWEN3_8B_LAYER = (
    ("qkv", 4096, 6144),
    ("o", 4096, 4096),
    ("gate_up", 4096, 24576),
    ("down", 12288, 4096),
)
QWEN3_8B_LAYERS = 36

# Skinny shapes standing in for the FlyDSL article's production list.
SKINNY_SHAPES = (
    ("k7168_n2112", 7168, 2112),
    ("k7168_n4096", 7168, 4096),
    ("k7168_n18432", 7168, 18432),
    ("k8192_n10240", 8192, 10240),
    ("k8192_n57344", 8192, 57344),
)


@dataclass(frozen=True)
class Case:
    name: str
    M: int
    N: int
    K: int
    seed: int = 0
    m_tile: int = 0


def config_single():
    """Single GEMM M=1, K=N=4096, seed 0."""
    return [Case("single_m1_4096x4096", 1, 4096, 4096, 0)]


def config_qwen3_decode(ms=(1, 2, 4, 8, 16)):
    """Qwen3-8B-shaped decode GEMMs at M in {1,2,4,8,16}."""
    return [Case(f"{name}_m{M}", M, N, K, 0) for M in ms for (name, K, N) in QWEN3_8B_LAYER]


def config_skinny(ms=(1, 4, 8)):
    """K=7168 / 8192 skinny shapes at M in {1,4,8}."""
    return [Case(f"{name}_m{M}", M, N, K, 0) for M in ms for (name, K, N) in SKINNY_SHAPES]


def config_l2_reuse(ms=(32, 64), m_tiles=(16, 32)):
    """gate_up and down at M in {32, 64} with M-tile 16 or 32 (0: all of M in
    one tile, for comparison)."""
    shapes = [s for s in QWEN3_8B_LAYER if s[0] in ("gate_up", "down")]
    return [Case(f"{name}_m{M}_tm{tm}", M, N, K, 0, tm)
            for M in ms for tm in m_tiles for (name, K, N) in shapes]


def chain_layout(layers: int = QWEN3_8B_LAYERS, M: int = 16):
    """Task list of the persistent chain: layers x (qkv, o, gate_up, down).
    Task t = 4*layer + g draws X with seed t and W with seed 10000 + t."""
    out = []
    for layer in range(layers):
        for g, (name, K, N) in enumerate(QWEN3_8B_LAYER):
            t = 4 * layer + g
            out.append(Case(f"L{layer}_{name}", M, N, K, t))
    return out


def _gen(seed: int, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_xw(M: int, N: int, K: int, seed: int = 0, device="cpu"):
    """X [M,K] ~ N(0,1) then W [N,K] ~ N(0,1/K) from one generator; bf16."""
    g = _gen(seed, device)
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    w = torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * (1.0 / K ** 0.5)
    return x.to(torch.bfloat16), w.to(torch.bfloat16)


def make_x(M: int, K: int, seed: int, device="cpu"):
    g = _gen(seed, device)
    return torch.randn(M, K, generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)


def make_w(N: int, K: int, seed: int, device="cpu"):
    g = _gen(seed, device)
    w = torch.randn(N, K, generator=g, dtype=torch.float32, device=device) * (1.0 / K ** 0.5)
    return w.to(torch.bfloat16)


def make_case(case: Case, device="cpu"):
    return make_xw(case.M, case.N, case.K, case.seed, device)


def make_int_xw(M: int, N: int, K: int, seed: int = 0, lo: int = -3, hi: int = 3):
    """Small-integer X, W (exact in bf16; every partial sum exact in fp32 while
    K * hi * hi < 2^24)."""
    g = _gen(seed)
    x = torch.randint(lo, hi + 1, (M, K), generator=g, dtype=torch.int32)
    w = torch.randint(lo, hi + 1, (N, K), generator=g, dtype=torch.int32)
    return x.to(torch.bfloat16), w.to(torch.bfloat16)


def make_permutation_w(N: int, seed: int = 0):
    """W = a permutation matrix [N, N] (bf16) and the permutation p, W[n, p[n]] = 1."""
    g = _gen(seed)
    p = torch.randperm(N, generator=g)
    w = torch.zeros(N, N, dtype=torch.bfloat16)
    w[torch.arange(N), p] = 1
    return w, p


def make_onehot_x(M: int, K: int, seed: int = 0):
    """X rows are one-hot [M, K] (bf16) and the hot index per row."""
    g = _gen(seed)
    idx = torch.randint(0, K, (M,), generator=g)
    x = torch.zeros(M, K, dtype=torch.bfloat16)
    x[torch.arange(M), idx] = 1
    return x, idx


def make_binade_xw(M: int, N: int, K: int, seed: int = 0, emin: int = -6, emax: int = 2):
    """Random bf16 with exponents in [emin, emax] and random sign/fraction: all
    products and sums of a small K are exact in fp64 (tiny brute-force cases)."""
    g = _gen(seed)

    def draw(shape):
        frac = torch.randint(0, 128, shape, generator=g, dtype=torch.int32)
        exp = torch.randint(emin, emax + 1, shape, generator=g, dtype=torch.int32)
        sign = torch.randint(0, 2, shape, generator=g, dtype=torch.int32) * 2 - 1
        val = sign.double() * (1.0 + frac.double() / 128.0) * torch.pow(2.0, exp.double())
        return val.to(torch.bfloat16)

    return draw((M, K)), draw((N, K))
