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
        """Attention forward FLOPs as the metric counts them: 2*B*Hq*T^2*d when
        causal (QK^T and PV over the causal half), 4*B*Hq*T^2*d otherwise."""
        return (2.0 if self.causal else 4.0) * self.B * self.Hq * self.T * self.T * self.d

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


@dataclass(frozen=True)
class DecodeWorkload:
    """One decode step of a serving batch over a paged K/V cache.

    Sequence lengths are drawn by a numpy ``default_rng(seed)`` as integers
    uniform in [1, max_len]; the cache is filled as make_paged does (q, then
    K, then V standard normal, Q and K times sigma_qk, rounded to bf16; blocks
    at a random permutation of the pool).
    """
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    bs: int
    max_len: int
    seed: int
    sigma_qk: float = 1.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def seq_lens(self) -> np.ndarray:
        rng = np.random.default_rng(self.seed)
        return rng.integers(1, self.max_len + 1, size=self.B).astype(np.int32)

    def io_bytes(self) -> int:
        """Bytes one step must move through HBM: the K and V rows of every cached
        token, q and o (bf16), lse (fp32), the lengths and the block ids used."""
        lens = self.seq_lens().astype(np.int64)
        kv = int(lens.sum()) * self.Hkv * self.d * 2 * 2
        qo = 2 * self.B * self.Hq * self.d * 2
        blocks = int(((lens + self.bs - 1) // self.bs).sum())
        return kv + qo + self.B * self.Hq * 4 + self.B * 4 + blocks * 4

    def describe(self) -> dict:
        out = asdict(self)
        out["G"] = self.G
        lens = self.seq_lens()
        out["tokens"] = int(lens.sum())
        return out


# The decode step measured beside the forward: the headline head configuration
# (Hq=32, Hkv=8, d=128) serving 64 sequences with contexts up to 16384 tokens.
DECODE = DecodeWorkload("decode_b64_hq32_hkv8_d128_bs16_len1to16384", B=64, Hq=32, Hkv=8,
                        d=128, bs=16, max_len=16384, seed=11)
# The same serving batch at head dimension 64.
DECODE_D64 = DecodeWorkload("decode_b64_hq32_hkv8_d64_bs16_len1to16384", B=64, Hq=32, Hkv=8,
                            d=64, bs=16, max_len=16384, seed=11)


def make_paged_device(w: DecodeWorkload, device, spare_blocks: int = 3):
    """make_paged's recipe for a decode workload, drawn on ``device`` (a CUDA
    generator seeded with w.seed; the block permutation comes from a CPU
    generator with the same seed); the table has ceil(max_len / bs) columns.
    Returns (q, k_cache, v_cache, block_table,
    seq_lens) as device tensors (table and lengths int32)."""
    lens = w.seq_lens()
    need = [(int(n) + w.bs - 1) // w.bs for n in lens]
    max_blocks = (w.max_len + w.bs - 1) // w.bs  # the table covers the longest context
    num_blocks = sum(need) + spare_blocks
    g = torch.Generator(device=device)
    g.manual_seed(int(w.seed))
    q = (torch.randn((w.B, w.Hq, w.d), generator=g, device=device) * w.sigma_qk).to(torch.bfloat16)
    caches = []
    for sigma in (w.sigma_qk, 1.0):
        c = torch.empty((num_blocks, w.Hkv, w.bs, w.d), dtype=torch.bfloat16, device=device)
        for i in range(0, num_blocks, 4096):  # in slices, to bound the fp32 temporary
            j = min(num_blocks, i + 4096)
            c[i:j] = (torch.randn((j - i, w.Hkv, w.bs, w.d), generator=g, device=device)
                      * sigma).to(torch.bfloat16)
        caches.append(c)
    gc = torch.Generator(device="cpu")
    gc.manual_seed(int(w.seed))
    perm = torch.randperm(num_blocks, generator=gc).numpy().astype(np.int32)
    table = np.full((w.B, max_blocks), -1, dtype=np.int32)
    pos = 0
    for b in range(w.B):
        table[b, :need[b]] = perm[pos:pos + need[b]]
        pos += need[b]
    return (q, caches[0], caches[1], torch.from_numpy(table).to(device),
            torch.from_numpy(lens).to(device))


def gather_sequences(table: np.ndarray, seq_lens: np.ndarray, rows, bs: int,
                     k_cache: torch.Tensor, v_cache: torch.Tensor):
    """A compact copy of the cache for the sequences ``rows``: their blocks,
    renumbered 0..n-1 in table order, and the matching table and lengths
    (host tensors).  Lets the oracle check selected sequences of a cache too
    large for it."""
    sub_lens = np.asarray(seq_lens, dtype=np.int32)[list(rows)]
    ids, sub_rows = [], []
    for b in rows:
        n = (int(seq_lens[b]) + bs - 1) // bs
        sub_rows.append(list(range(len(ids), len(ids) + n)))
        ids += [int(x) for x in table[b, :n]]
    max_blocks = max([len(r) for r in sub_rows] + [1])
    sub_table = np.full((len(rows), max_blocks), -1, dtype=np.int32)
    for i, r in enumerate(sub_rows):
        sub_table[i, :len(r)] = r
    idx = torch.tensor(ids if ids else [0], dtype=torch.long, device=k_cache.device)
    return (k_cache.index_select(0, idx).cpu(), v_cache.index_select(0, idx).cpu(), sub_table,
            sub_lens)


def make_packed(lens, Hq: int, Hkv: int, d: int, seed: int, sigma_qk: float = 1.0):
    """Packed sequences for the variable-length forward: (q [total, Hq, d],
    k, v [total, Hkv, d]) bf16 CPU tensors and cu_seqlens int32 [B+1] (numpy).
    A torch CPU generator seeded with ``seed`` draws q, then k, then v
    standard normal in row-major order; q and k are multiplied by sigma_qk."""
    lens = [int(n) for n in lens]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((total, Hq, d), generator=g) * sigma_qk
    k = torch.randn((total, Hkv, d), generator=g) * sigma_qk
    v = torch.randn((total, Hkv, d), generator=g)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), cu


@dataclass(frozen=True)
class VarlenWorkload:
    """A packed batch of mixed-length sequences (lengths uniform in
    [min_len, max_len] from numpy default_rng(seed)), drawn as make_packed."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    min_len: int
    max_len: int
    seed: int

    def lens(self) -> list:
        rng = np.random.default_rng(self.seed)
        return [int(x) for x in rng.integers(self.min_len, self.max_len + 1, size=self.B)]

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    @property
    def flops(self) -> float:
        """The metric's causal count per sequence, summed: 2*Hq*T_b^2*d."""
        return float(sum(2.0 * self.Hq * n * n * self.d for n in self.lens()))

    def describe(self) -> dict:
        out = asdict(self)
        lens = self.lens()
        out["total"] = int(sum(lens))
        out["longest"] = int(max(lens))
        return out


# Packed mixed lengths with the headline head configuration.
VARLEN = VarlenWorkload("varlen_b32_hq32_hkv8_d128_len128to8192", B=32, Hq=32, Hkv=8, d=128,
                        min_len=128, max_len=8192, seed=13)
