"""Parity of the packed variable-length forward with the fp64 oracle, through
the C ABI, on a B200.

Tolerance: the forward's (the per-sequence arithmetic is the forward's):
O max |err| <= 2e-2, mean <= 2e-3; LSE |err| <= 1e-3.

* small packed batches (lengths 0, 1, 127, 128, 129, 300, 1000 mixed; G = 1, 3,
  4; d = 64 and 128; causal and full): every element;
* a serving-like mix of long sequences: sampled rows;
* equal lengths: the same bits as tessera_attn_fwd on the padded batch;
* rows of skipped or absent sequences untouched; offsets out of range
  reported.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    tess.load_library()
    assert tess.tessera_attn_device_error() == 0


def check(o, lse, ro, rlse, what, rows=None):
    o = o.double().numpy()
    lse = lse.double().numpy()
    if rows is not None:
        o, ro = o[rows], ro[rows]
        lse, rlse = lse[:, rows], rlse[:, rows]
    err = np.abs(o - ro)
    assert np.all(np.isfinite(o)), what
    assert err.max() <= 2e-2, f"{what}: O max {err.max():.3e}"
    assert err.mean() <= 2e-3, f"{what}: O mean {err.mean():.3e}"
    assert np.abs(lse - rlse).max() <= 1e-3, f"{what}: LSE {np.abs(lse - rlse).max():.3e}"


def run(lens, Hq, Hkv, d, causal, seed, sigma=1.5):
    q, k, v, cu = inputs.make_packed(lens, Hq, Hkv, d, seed=seed, sigma_qk=sigma)
    cu_d = torch.from_numpy(cu).to(DEV)
    o, lse = tess.attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu_d, max(lens + [0]),
                                  causal=causal)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    return q, k, v, cu, o.float().cpu(), lse.cpu()


CASES = [
    ([1, 127, 128, 129], 4, 2, 64, True),
    ([300, 0, 1000, 17], 8, 2, 128, True),
    ([513, 255], 6, 2, 128, True),       # G = 3
    ([200, 700, 1], 4, 4, 64, True),     # G = 1
    ([100, 333], 8, 2, 128, False),      # full attention: keys past a sequence masked
    ([129], 2, 1, 64, False),
]


@pytest.mark.parametrize("lens,Hq,Hkv,d,causal", CASES)
def test_varlen_every_element(lens, Hq, Hkv, d, causal):
    q, k, v, cu, o, lse = run(lens, Hq, Hkv, d, causal, seed=700 + sum(lens) + d)
    assert tess.tessera_attn_last_launch_count() == 1
    ro, rlse = oracle.attn_fwd_varlen_f64(q.double().numpy(), k.double().numpy(),
                                          v.double().numpy(), cu, causal=causal,
                                          scale=1.0 / math.sqrt(d))
    check(o, lse, ro, rlse, (lens, Hq, Hkv, d, causal))


def test_varlen_long_mix_sampled_rows():
    lens = [4096, 37, 2048, 3000, 128, 1]
    Hq, Hkv, d = 32, 8, 128
    q, k, v, cu, o, lse = run(lens, Hq, Hkv, d, True, seed=11, sigma=4.0)
    total = int(cu[-1])
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([rng.choice(total, 40, replace=False),
                                     cu[:-1], np.maximum(cu[1:] - 1, 0)]))
    rows = rows[rows < total]
    # oracle rows one by one, each within its own sequence (rows entry point
    # on that sequence viewed as a [1, H, T_b, d] batch)
    ro = np.zeros((total, Hq, d))
    rlse = np.zeros((Hq, total))
    for b in range(len(lens)):
        s, e = int(cu[b]), int(cu[b + 1])
        mine = rows[(rows >= s) & (rows < e)]
        if len(mine) == 0:
            continue
        view = lambda x: inputs.bf16_bits(x[s:e].permute(1, 0, 2).contiguous()[None])
        sel = np.array([(0, h, r - s) for r in mine for h in range(Hq)], dtype=np.int64)
        orow, lrow = oracle.attn_rows_bf16(view(q), view(k), view(v), sel, causal=True,
                                           scale=1.0 / math.sqrt(d))
        for n, (r, h) in enumerate((r, h) for r in mine for h in range(Hq)):
            ro[r, h] = orow[n]
            rlse[h, r] = lrow[n]
    check(o, lse, ro, rlse, "long mix", rows=rows)


def test_varlen_equal_lengths_match_fixed_length_bits():
    B, T, Hq, Hkv, d = 3, 1000, 8, 2, 128
    q, k, v = (t.to(DEV) for t in inputs.make_qkv(B, Hq, Hkv, T, d, seed=12))
    of, lf = tess.attn_fwd(q, k, v, causal=True)
    pack = lambda x: x.permute(0, 2, 1, 3).reshape(B * T, x.shape[1], d).contiguous()
    cu = torch.arange(B + 1, dtype=torch.int32, device=DEV) * T
    ov, lv = tess.attn_fwd_varlen(pack(q), pack(k), pack(v), cu, T, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(ov, pack(of))
    assert torch.equal(lv, lf.permute(1, 0, 2).reshape(Hq, B * T))


def test_varlen_bad_offsets_are_reported_and_skipped():
    lens = [300, 200, 100]
    Hq, Hkv, d = 4, 2, 64
    q, k, v, cu = inputs.make_packed(lens, Hq, Hkv, d, seed=13)
    total = int(cu[-1])
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    good_o, good_l = tess.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(cu).to(DEV), 300)
    torch.cuda.synchronize()
    # sequence 1 given as longer than max_seqlen: skipped, the others bit-exact
    bad = cu.copy()
    bad[2] = bad[1] + 301
    bad[3] = total
    o = torch.full_like(qd, 7.0)
    lse = torch.full((Hq, total), 7.0, device=DEV)
    tess.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(bad).to(DEV), 300, out=o, lse=lse)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_VARLEN_INPUT
    s1, e1 = int(cu[1]), int(cu[1]) + 301
    assert torch.all(o[s1:min(e1, total)] == 7.0)
    assert torch.equal(o[:s1], good_o[:s1])
    # offsets out of order: that sequence skipped
    bad = cu.copy()
    bad[1], bad[2] = bad[2], bad[1]
    tess.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(bad).to(DEV), 300)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_VARLEN_INPUT
    # and a clean call afterwards
    o2, _ = tess.attn_fwd_varlen(qd, kd, vd, torch.from_numpy(cu).to(DEV), 300)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    assert torch.equal(o2, good_o)


def test_varlen_empty_sequences_leave_nothing_behind():
    lens = [0, 0, 50, 0]
    Hq, Hkv, d = 2, 1, 64
    q, k, v, cu = inputs.make_packed(lens, Hq, Hkv, d, seed=14)
    o = torch.full((50, Hq, d), 7.0, dtype=torch.bfloat16, device=DEV)
    tess.attn_fwd_varlen(q.to(DEV), k.to(DEV), v.to(DEV), torch.from_numpy(cu).to(DEV), 50,
                         out=o)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    ro, _ = oracle.attn_fwd_varlen_f64(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy(), cu, scale=1.0 / math.sqrt(d))
    assert np.abs(o.float().cpu().numpy() - ro).max() <= 2e-2
