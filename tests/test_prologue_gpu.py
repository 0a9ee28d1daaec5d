"""Parity of the CUDA prologue kernels (RMSNorm; rotary embedding with the
head split) with the fp64 oracle, through the C ABI, on a B200.

Tolerance: both kernels compute in fp32 from bf16 inputs and round the
result to bf16 once (relative 2^-8 at most).  Written in the tests below:
RMSNorm |y - ref| <= 2^-8 |ref| + 1e-6 (the fp32 sum of squares and the
reciprocal square root add a few fp32 ulps); RoPE |y - ref| <= 2^-8 |ref| +
1e-5 (|x_i| + |x_{i+d/2}|) (fp32 products and fp32-rounded cos/sin); value
heads and position 0 exactly.  The chained prologue -> attention check uses
the forward's tolerance on O (max 2e-2, mean 2e-3) since every step rounds to
bf16 as the product path does.
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


def _bf16(shape, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * sigma).to(torch.bfloat16)


def check_norm(y, ref, what):
    y = y.double().numpy()
    err = np.abs(y - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-6
    assert np.all(err <= bound), f"{what}: worst excess {(err - bound).max():.3e}"


@pytest.mark.parametrize("rows,dim,eps,sigma", [
    (1, 8, 1e-6, 1.0), (5, 64, 1e-6, 1.0), (33, 4096, 1e-5, 1.0), (7, 8192, 1e-6, 3.0),
    (100, 1000, 1e-6, 0.01), (300, 256, 0.5, 0.2), (17, 2048, 0.0, 10.0),
])
def test_rmsnorm_every_element(rows, dim, eps, sigma):
    x = _bf16((rows, dim), 100 + dim, sigma)
    w = _bf16((dim,), 200 + dim)
    y = tess.rmsnorm(x.to(DEV), w.to(DEV), eps)
    torch.cuda.synchronize()
    assert tess.tessera_attn_last_launch_count() == 1
    ref = oracle.rmsnorm_f64(x.double().numpy(), w.double().numpy(), eps)
    check_norm(y.cpu(), ref, (rows, dim, eps))


def test_rmsnorm_in_place_and_large_rows_sampled():
    rows, dim = 16384, 4096
    x = _bf16((rows, dim), 7)
    w = _bf16((dim,), 8)
    xd, wd = x.to(DEV), w.to(DEV)
    y = tess.rmsnorm(xd, wd, 1e-6)
    xin = xd.clone()
    tess.rmsnorm(xin, wd, 1e-6, out=xin)  # in place
    torch.cuda.synchronize()
    assert torch.equal(y, xin)
    sel = np.random.default_rng(3).choice(rows, 64, replace=False)
    sel = np.unique(np.concatenate([sel, [0, rows - 1]]))
    ref = oracle.rmsnorm_f64(x[sel].double().numpy(), w.double().numpy(), 1e-6)
    check_norm(y[sel].cpu(), ref, "sampled rows")


@pytest.mark.parametrize("dim", [4096, 8192])
def test_rmsnorm_wide_rows_guard_regions_and_odd_counts(dim):
    # wide rows go through shared memory by bulk copy: fewer rows than the
    # grid's warps, an odd count, and untouched memory on both sides of y
    pad = 64
    for rows in (1, 5, 4097):
        x = _bf16((rows, dim), 300 + rows, 1.5)
        w = _bf16((dim,), 301)
        buf = torch.full((rows * dim + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
        out = buf[pad:pad + rows * dim].view(rows, dim)
        tess.rmsnorm(x.to(DEV), w.to(DEV), 1e-6, out=out)
        torch.cuda.synchronize()
        assert tess.tessera_attn_device_error() == 0
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
        sel = np.unique(np.r_[0, rows - 1, np.arange(0, rows, max(1, rows // 7))])
        ref = oracle.rmsnorm_f64(x[sel].double().numpy(), w.double().numpy(), 1e-6)
        check_norm(out[sel].cpu(), ref, (rows, dim))


def test_rmsnorm_zero_row_and_guard_regions():
    dim = 512
    x = torch.zeros((3, dim), dtype=torch.bfloat16)
    x[1] = _bf16((dim,), 9)
    w = _bf16((dim,), 10)
    pad = 4096
    buf = torch.full((3 * dim + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    out = buf[pad:pad + 3 * dim].view(3, dim)
    tess.rmsnorm(x.to(DEV), w.to(DEV), 1e-6, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 7.0) and torch.all(buf[-pad:] == 7.0)
    assert not out[0].any() and not out[2].any()  # 0 * rsqrt(eps) * w = 0
    ref = oracle.rmsnorm_f64(x.double().numpy(), w.double().numpy(), 1e-6)
    check_norm(out.cpu(), ref, "zero rows")


def check_rope(got, ref, x_pairs, what):
    got = got.double().numpy()
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * x_pairs
    assert np.all(err <= bound), f"{what}: worst excess {(err - bound).max():.3e}"


def _pair_mag(heads):
    """|x_i| + |x_{i+d/2}| laid out like the rotated output ([B,H,T,d])."""
    h = np.abs(heads.double().numpy())
    half = h.shape[-1] // 2
    s = h[..., :half] + h[..., half:]
    return np.concatenate([s, s], axis=-1).transpose(0, 2, 1, 3)


@pytest.mark.parametrize("B,T,Hq,Hkv,d,base,pos_kind", [
    (1, 1, 1, 1, 64, 10000.0, None), (2, 37, 4, 2, 128, 10000.0, None),
    (1, 100, 8, 8, 64, 10000.0, "random"), (3, 17, 6, 2, 128, 500000.0, "random"),
    (2, 300, 32, 8, 128, 10000.0, None), (1, 16, 4, 1, 128, 10000.0, "offset"),
])
def test_rope_every_element(B, T, Hq, Hkv, d, base, pos_kind):
    H3 = Hq + 2 * Hkv
    qkv = _bf16((B, T, H3 * d), 300 + T + d, 2.0)
    pos = None
    if pos_kind == "random":
        pos = np.random.default_rng(T).integers(0, 200000, size=(B, T)).astype(np.int32)
    elif pos_kind == "offset":  # a decode-like continuation: positions 5000 + t
        pos = (5000 + np.tile(np.arange(T), (B, 1))).astype(np.int32)
    pos_d = torch.from_numpy(pos).to(DEV) if pos is not None else None
    q, k, v = tess.rope_qkv(qkv.to(DEV), Hq, Hkv, positions=pos_d, base=base)
    torch.cuda.synchronize()
    assert tess.tessera_attn_last_launch_count() == 1
    rq, rk, rv = oracle.rope_qkv_f64(qkv.double().numpy(), Hq, Hkv, positions=pos, base=base)
    heads = qkv.reshape(B, T, H3, d)
    check_rope(q.cpu(), rq, _pair_mag(heads[:, :, :Hq]), "q")
    check_rope(k.cpu(), rk, _pair_mag(heads[:, :, Hq:Hq + Hkv]), "k")
    assert torch.equal(v.cpu(), heads[:, :, Hq + Hkv:].permute(0, 2, 1, 3).contiguous())


def test_rope_position_zero_is_exact_identity():
    B, T, Hq, Hkv, d = 2, 40, 4, 2, 128
    qkv = _bf16((B, T, (Hq + 2 * Hkv) * d), 11)
    pos = torch.zeros((B, T), dtype=torch.int32, device=DEV)
    q, k, v = tess.rope_qkv(qkv.to(DEV), Hq, Hkv, positions=pos)
    torch.cuda.synchronize()
    heads = qkv.reshape(B, T, Hq + 2 * Hkv, d).permute(0, 2, 1, 3)
    assert torch.equal(q.cpu(), heads[:, :Hq].contiguous())
    assert torch.equal(k.cpu(), heads[:, Hq:Hq + Hkv].contiguous())


def test_rope_headline_shape_sampled_tokens():
    # the headline attention configuration: 16384 tokens, Hq=32, Hkv=8, d=128
    B, T, Hq, Hkv, d = 1, 16384, 32, 8, 128
    H3 = Hq + 2 * Hkv
    qkv = _bf16((B, T, H3 * d), 12)
    q, k, v = tess.rope_qkv(qkv.to(DEV), Hq, Hkv)
    torch.cuda.synchronize()
    sel = np.unique(np.concatenate([np.random.default_rng(4).choice(T, 48, replace=False),
                                    [0, 1, 15, 16, T - 1]]))
    sub = qkv[:, sel]
    pos = np.asarray(sel, dtype=np.int32)[None, :]
    rq, rk, rv = oracle.rope_qkv_f64(sub.double().numpy(), Hq, Hkv, positions=pos)
    heads = sub.reshape(B, len(sel), H3, d)
    check_rope(q[:, :, sel].cpu(), rq, _pair_mag(heads[:, :, :Hq]), "q sampled")
    check_rope(k[:, :, sel].cpu(), rk, _pair_mag(heads[:, :, Hq:Hq + Hkv]), "k sampled")
    assert torch.equal(v[:, :, sel].cpu(), heads[:, :, Hq + Hkv:].permute(0, 2, 1, 3))


def test_prologue_chain_into_attention():
    """hidden states -> RMSNorm -> projection (a plain GEMM, here torch's, as
    the model would run it) -> RoPE -> attention, against the same chain in
    the oracle (fp64, with the product path's bf16 roundings between steps)."""
    B, T, Hq, Hkv, d = 2, 160, 4, 2, 64
    Dm = Hq * d
    H3 = Hq + 2 * Hkv
    x = _bf16((B, T, Dm), 21)
    wn = (1.0 + 0.1 * _bf16((Dm,), 22).float()).to(torch.bfloat16)
    wqkv = (_bf16((Dm, H3 * d), 23).float() / math.sqrt(Dm)).to(torch.bfloat16)
    h = tess.rmsnorm(x.to(DEV), wn.to(DEV), 1e-6)
    qkv = (h @ wqkv.to(DEV)).contiguous()
    q, k, v = tess.rope_qkv(qkv, Hq, Hkv)
    o, lse = tess.attn_fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    # oracle chain, rounding to bf16 where the product path stores bf16
    hr = torch.from_numpy(oracle.rmsnorm_f64(x.double().numpy(), wn.double().numpy(), 1e-6))
    hr = hr.to(torch.bfloat16).double()
    qkvr = (hr @ wqkv.double()).to(torch.bfloat16).double()
    rq, rk, rv = oracle.rope_qkv_f64(qkvr.numpy(), Hq, Hkv)
    rq, rk, rv = (torch.from_numpy(a).to(torch.bfloat16).double().numpy() for a in (rq, rk, rv))
    ro, rlse = oracle.attn_fwd_f64(rq, rk, rv, causal=True, scale=1.0 / math.sqrt(d))
    err = np.abs(o.float().cpu().double().numpy() - ro)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert np.abs(lse.cpu().double().numpy() - rlse).max() <= 1e-2
