"""Seeded synthetic inputs for causal grouped-query attention.

This module only draws random numbers and holds the workload table; it does no
attention arithmetic.  Both the CUDA path and the fp64 oracle are fed from it.

Recipe (the same for every workload): a torch CPU ``Generator`` seeded with the
workload's seed draws standard-normal fp32 samples for Q, then K, then V, in
that order and in row-major [B,H,T,d] order; Q and K are multiplied by
``sigma_qk`` (V by 1) and each tensor is rounded to bf16 (round to nearest
even).  Because Q is drawn first, workloads that share a seed and Q's shape
share Q exactly (the GQA group sweep relies on this).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    d: int
    seed: int
    sigma_qk: float = 1.0
    causal: bool = True

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    @property
    def flops(self) -> float:
        """Causal attention forward FLOPs as the metric counts them: 2*B*Hq*T^2*d."""
        return 2.0 * self.B * self.Hq * self.T * self.T * self.d

    @property
    def io_bytes(self) -> int:
        """Bytes that must cross HBM once: Q, K, V, O in bf16 and LSE in fp32."""
        q = self.B * self.Hq * self.T * self.d * 2
        kv = 2 * self.B * self.Hkv * self.T * self.d * 2
        return q + kv + q + self.B * self.Hq * self.T * 4

    def describe(self) -> dict:
        out = asdict(self)
        out["G"] = self.G
        return out


# The seven synthetic workloads: causal attention, Q/K/V bf16 i.i.d. normal.
WORKLOADS = {
    w.name: w for w in [
        Workload("b2_t128_hq4_hkv2_d64", B=2, T=128, Hq=4, Hkv=2, d=64, seed=0),
        Workload("b8_t1000_hq8_hkv2_d64", B=8, T=1000, Hq=8, Hkv=2, d=64, seed=1),
        Workload("b4_t4096_hq16_hkv4_d128", B=4, T=4096, Hq=16, Hkv=4, d=128, seed=2),
        Workload("b1_t16384_hq32_hkv8_d128_sigma4", B=1, T=16384, Hq=32, Hkv=8,
                 d=128, seed=3, sigma_qk=4.0),
        Workload("b8_t2048_hq32_hkv32_d128_mha", B=8, T=2048, Hq=32, Hkv=32, d=128, seed=4),
        Workload("b8_t2048_hq32_hkv8_d128_gqa", B=8, T=2048, Hq=32, Hkv=8, d=128, seed=4),
        Workload("b8_t2048_hq32_hkv1_d128_mqa", B=8, T=2048, Hq=32, Hkv=1, d=128, seed=4),
    ]
}

SMALL = "b2_t128_hq4_hkv2_d64"
TAIL = "b8_t1000_hq8_hkv2_d64"
LARGEST = "b1_t16384_hq32_hkv8_d128_sigma4"


def make_qkv(B: int, Hq: int, Hkv: int, T: int, d: int, seed: int,
             sigma_qk: float = 1.0):
    """Draw (q, k, v) as bf16 CPU tensors, q [B,Hq,T,d], k and v [B,Hkv,T,d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Hq, T, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Hkv, T, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, T, d), generator=g, dtype=torch.float32)
    if sigma_qk != 1.0:
        q.mul_(sigma_qk)
        k.mul_(sigma_qk)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


# The upstream gradient dO of a workload draws from its own generator, seeded
# with the workload's seed plus this offset, so Q/K/V stay the forward's.
GRAD_SEED_OFFSET = 1_000_003


def make_grad(B: int, Hq: int, T: int, d: int, seed: int):
    """Draw dO as a bf16 CPU tensor [B,Hq,T,d] of standard normals."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn((B, Hq, T, d), generator=g, dtype=torch.float32).to(torch.bfloat16)


def workload_grad(w: Workload | str):
    """dO for a workload: make_grad with the workload's seed + GRAD_SEED_OFFSET."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    return make_grad(w.B, w.Hq, w.T, w.d, w.seed + GRAD_SEED_OFFSET)


def workload_inputs(w: Workload | str):
    """Inputs of a named workload (bf16 CPU tensors)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    return make_qkv(w.B, w.Hq, w.Hkv, w.T, w.d, w.seed, w.sigma_qk)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bit patterns of a bf16 CPU tensor as a uint16 numpy array."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def sample_rows(B: int, Hq: int, T: int, n: int, seed: int) -> np.ndarray:
    """(b, h, i) triples to check on workloads too large for a full oracle run.

    Always includes the first and last rows of every 128-row tile boundary
    neighbourhood for a few heads (rows 0, 1, 127, 128, 129, T-2, T-1) and
    fills the rest uniformly at random.  Sorted by (b, h, i).
    """
    rng = np.random.default_rng(seed)
    fixed_i = sorted({i for i in (0, 1, 127, 128, 129, 255, 256, T // 2, T - 2, T - 1)
                      if 0 <= i < T})
    rows = set()
    for bh in {(0, 0), (B - 1, Hq - 1), (0, Hq - 1), (B - 1, 0)}:
        for i in fixed_i:
            rows.add((bh[0], bh[1], i))
    total = B * Hq * T
    while len(rows) < min(n, total):
        rows.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(T))))
    return np.array(sorted(rows), dtype=np.int64)


def make_paged(B: int, Hq: int, Hkv: int, d: int, bs: int, seq_lens, seed: int,
               spare_blocks: int = 3, sigma_qk: float = 1.0):
    """A decode step over a paged cache: (q [B,Hq,d], k_cache, v_cache
    [num_blocks,Hkv,bs,d] bf16, block_table int32 [B,max_blocks], seq_lens int32 [B]).

    Each sequence gets ceil(len/bs) blocks at random physical positions (a
    random permutation of the pool, which has spare_blocks unused blocks);
    unused table entries are -1.
    """
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    need = [(int(n) + bs - 1) // bs for n in seq_lens]
    max_blocks = max(need + [1])
    num_blocks = sum(need) + spare_blocks
    q = torch.randn((B, Hq, d), generator=g, dtype=torch.float32) * sigma_qk
    k = torch.randn((num_blocks, Hkv, bs, d), generator=g, dtype=torch.float32) * sigma_qk
    v = torch.randn((num_blocks, Hkv, bs, d), generator=g, dtype=torch.float32)
    perm = torch.randperm(num_blocks, generator=g).numpy().astype(np.int32)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    pos = 0
    for b in range(B):
        table[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), table, seq_lens)
