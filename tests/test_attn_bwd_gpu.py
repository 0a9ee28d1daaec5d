"""Parity of the CUDA backward (dQ, dK, dV) with the fp64 oracle, through the
C ABI, on a B200.

The forward's O and LSE come from the CUDA forward (the product path runs
forward then backward); every expected value comes from the oracle, which
recomputes the forward itself from Q, K, V and dO.

Tolerance (stated for this path; the arithmetic keeps P and dS in bf16 for
the MMAs and rounds the outputs to bf16, each a relative 2^-9): for each of
dQ, dK, dV, with R = max |reference| over the compared elements,
max |err| <= 2.5e-2 * R and mean |err| <= 2.5e-3 * R.

* small shapes and the two smallest synthetic workloads: every element;
* the T = 4096 workload: every element of dQ, dK and dV against the oracle's
  full backward, its (batch, K/V head) slices run on every host core;
* the larger workloads: sampled dQ rows computed one by one by the oracle, and
  properties that hold at any size (sum_j dV[j] equals the group's summed dO;
  sum_j dK[j] = 0), checked in fp64 on the GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu

REL_MAX = 2.5e-2
REL_MEAN = 2.5e-3


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    tess.load_library()
    assert tess.tessera_attn_device_error() == 0


def run_gpu_bwd(q, k, v, g, causal, scale):
    """bf16 CPU tensors in; (dq, dk, dv) fp32 CPU out, via the forward's O/LSE."""
    dev = torch.device("cuda:0")
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    o, lse = tess.attn_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = tess.attn_bwd(qd, kd, vd, o, lse, gd, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert tess.tessera_attn_last_launch_count() == expected_launches(q.shape, k.shape[1])
    assert tess.tessera_attn_device_error() == 0
    return dq.float().cpu(), dk.float().cpu(), dv.float().cpu()


def expected_launches(qshape, Hkv):
    """3, or 4 when the library's balanced dK/dV form applies to the shape
    (its workspace query asks for more than D)."""
    B, Hq, T, d = qshape
    balanced = (tess.tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)
                > tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d))
    return 4 if balanced else 3


def check_grad(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), what
    R = max(np.max(np.abs(ref)), 1e-30)
    err = np.abs(got - ref)
    assert err.max() <= REL_MAX * R, f"{what}: max err {err.max():.3e} vs R {R:.3e}"
    assert err.mean() <= REL_MEAN * R, f"{what}: mean err {err.mean():.3e} vs R {R:.3e}"
    return float(err.max() / R), float(err.mean() / R)


def oracle_bwd(q, k, v, g, causal, scale):
    return oracle.attn_bwd_f64(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               g.double().numpy(), causal=causal, scale=scale)


# (B, Hq, Hkv, T, d, causal): tails, single tiles, G odd / even / 1, full attention
SMALL = [
    (1, 2, 1, 1, 64, True), (2, 4, 2, 63, 64, True), (1, 2, 2, 128, 128, True),
    (1, 4, 1, 129, 64, True), (1, 3, 3, 200, 128, True), (2, 8, 2, 256, 64, True),
    (1, 6, 2, 300, 128, True), (1, 4, 2, 100, 64, False), (1, 2, 1, 129, 128, False),
    (1, 3, 1, 385, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,T,d,causal", SMALL)
def test_bwd_small_shapes_every_element(B, Hq, Hkv, T, d, causal):
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=2000 + T + d, sigma_qk=1.5)
    g = inputs.make_grad(B, Hq, T, d, seed=3000 + T)
    scale = 1.0 / math.sqrt(d)
    got = run_gpu_bwd(q, k, v, g, causal, scale)
    ref = oracle_bwd(q, k, v, g, causal, scale)
    for name, a, r in zip(("dQ", "dK", "dV"), got, ref):
        check_grad(a.numpy(), r, f"{name} {(B, Hq, Hkv, T, d, causal)}")


@pytest.mark.parametrize("name", [inputs.SMALL, inputs.TAIL])
def test_bwd_small_workloads_every_element(name):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    g = inputs.workload_grad(w)
    got = run_gpu_bwd(q, k, v, g, True, w.scale)
    ref = oracle_bwd(q, k, v, g, True, w.scale)
    for gname, a, r in zip(("dQ", "dK", "dV"), got, ref):
        check_grad(a.numpy(), r, f"{gname} {name}")


LARGE = [n for n in inputs.WORKLOADS if n not in (inputs.SMALL, inputs.TAIL)]
FULL_BWD = "b4_t4096_hq16_hkv4_d128"


def test_bwd_t4096_workload_every_element(parity_log):
    import time
    w = inputs.WORKLOADS[FULL_BWD]
    q, k, v = inputs.workload_inputs(w)
    g = inputs.workload_grad(w)
    got = run_gpu_bwd(q, k, v, g, True, w.scale)
    t0 = time.perf_counter()
    ref = oracle.attn_bwd_threaded(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                   g.double().numpy(), causal=True, scale=w.scale)
    el = time.perf_counter() - t0
    for gname, a, r in zip(("dQ", "dK", "dV"), got, ref):
        rmax, rmean = check_grad(a.numpy(), r, f"{gname} {FULL_BWD}")
        parity_log(test="backward every element", workload=FULL_BWD, grad=gname,
                   max_err_over_R=rmax, mean_err_over_R=rmean, elements=int(r.size),
                   oracle_s=round(el, 1), oracle_threads=oracle.host_threads())


@pytest.mark.parametrize("name", LARGE)
def test_bwd_large_workloads_sampled_rows_and_sums(name):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    g = inputs.workload_grad(w)
    dq, dk, dv = run_gpu_bwd(q, k, v, g, True, w.scale)
    rows = inputs.sample_rows(w.B, w.Hq, w.T, 64, seed=w.seed + 5)
    rq = oracle.attn_bwd_dq_rows_bf16(inputs.bf16_bits(q), inputs.bf16_bits(k),
                                      inputs.bf16_bits(v), inputs.bf16_bits(g), rows,
                                      causal=True, scale=w.scale)
    b, h, i = rows.T
    check_grad(dq[b, h, i].numpy(), rq, f"dQ rows {name}")
    # sum_j dV[b,g,j] = sum over the group's heads and rows of dO; sum_j dK = 0
    G = w.Hq // w.Hkv
    dev = torch.device("cuda:0")
    want = g.to(dev).double().reshape(w.B, w.Hkv, G, w.T, w.d).sum(dim=(2, 3))
    sv = dv.to(dev).double().sum(dim=2)
    scale_v = dv.to(dev).double().abs().sum(dim=2) + want.abs()
    assert torch.all((sv - want).abs() <= 1e-2 * scale_v + 1e-3), f"sum dV {name}"
    sk = dk.to(dev).double().sum(dim=2)
    assert torch.all(sk.abs() <= 1e-2 * dk.to(dev).double().abs().sum(dim=2) + 1e-3), \
        f"sum dK {name}"


def test_bwd_one_key_and_zero_gradient():
    B, Hq, Hkv, T, d = 2, 4, 2, 1, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=31)
    g = inputs.make_grad(B, Hq, T, d, seed=32)
    dq, dk, dv = run_gpu_bwd(q, k, v, g, True, 0.1)
    # P = 1, so dS = P * (dP - D) = 0 up to the rounding of dP (MMA) against D
    # (fp32 dot product) and of P recomputed from LSE
    assert dq.abs().max() <= 1e-4 and dk.abs().max() <= 1e-4
    want = g.float().reshape(B, Hkv, 2, T, d).sum(dim=2)
    assert torch.allclose(dv, want, rtol=1e-2, atol=1e-2)
    q, k, v = inputs.make_qkv(1, 4, 1, 300, 64, seed=33)
    dq, dk, dv = run_gpu_bwd(q, k, v, torch.zeros_like(q), True, 0.125)
    assert not dq.any() and not dk.any() and not dv.any()


def test_bwd_guard_regions_untouched():
    B, Hq, Hkv, T, d = 1, 4, 2, 200, 64
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in inputs.make_qkv(B, Hq, Hkv, T, d, seed=41))
    g = inputs.make_grad(B, Hq, T, d, seed=42).to(dev)
    o, lse = tess.attn_fwd(q, k, v)
    pad = 4096
    bufs = {}
    for name, like in (("dq", q), ("dk", k), ("dv", v)):
        big = torch.full((like.numel() + 2 * pad,), 7.0, dtype=torch.bfloat16, device=dev)
        bufs[name] = big
    views = {n: b[pad:pad + (q if n == "dq" else k).numel()].view((q if n == "dq" else k).shape)
             for n, b in bufs.items()}
    tess.attn_bwd(q, k, v, o, lse, g, dq=views["dq"], dk=views["dk"], dv=views["dv"])
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    for b in bufs.values():
        assert torch.all(b[:pad] == 7.0) and torch.all(b[-pad:] == 7.0)


@pytest.mark.parametrize("B,Hq,Hkv,T,d", [(1, 8, 2, 513, 128), (2, 4, 4, 300, 64),
                                           (1, 32, 1, 1000, 128)])
def test_bwd_repeated_calls_bitwise(B, Hq, Hkv, T, d):
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in inputs.make_qkv(B, Hq, Hkv, T, d, seed=51))
    g = inputs.make_grad(B, Hq, T, d, seed=52).to(dev)
    o, lse = tess.attn_fwd(q, k, v)
    a = [t.clone() for t in tess.attn_bwd(q, k, v, o, lse, g)]
    b = tess.attn_bwd(q, k, v, o, lse, g)
    torch.cuda.synchronize()
    # every gradient is summed in a fixed order (no atomics): the same bits on
    # every call, whatever the CTAs' timing
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("B,Hq,Hkv,T,d", [(1, 8, 1, 1000, 128), (2, 6, 3, 300, 64),
                                           (1, 32, 1, 2048, 128)])
def test_bwd_balanced_form_matches_three_kernel_form(B, Hq, Hkv, T, d):
    """Few key/value units: the split dK/dV units (fourth launch) against the
    three-kernel form forced by a workspace of D only.  dQ does not depend on
    the split (bit for bit); dK and dV differ only in the rounding of their
    sums."""
    dev = torch.device("cuda:0")
    q, k, v = (t.to(dev) for t in inputs.make_qkv(B, Hq, Hkv, T, d, seed=81, sigma_qk=1.5))
    g = inputs.make_grad(B, Hq, T, d, seed=82).to(dev)
    o, lse = tess.attn_fwd(q, k, v)
    assert (tess.tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)
            > tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d))
    bal = [t.clone() for t in tess.attn_bwd(q, k, v, o, lse, g)]
    assert tess.tessera_attn_last_launch_count() == 4
    small = torch.empty(tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d) // 4,
                        dtype=torch.float32, device=dev)
    three = tess.attn_bwd(q, k, v, o, lse, g, workspace=small)
    torch.cuda.synchronize()
    assert tess.tessera_attn_last_launch_count() == 3
    assert tess.tessera_attn_device_error() == 0
    assert torch.equal(bal[0], three[0])
    for a, b in zip(bal[1:], three[1:]):
        a, b = a.float(), b.float()
        R = b.abs().max().item()
        assert (a - b).abs().max().item() <= 2 ** -7 * R
    again = tess.attn_bwd(q, k, v, o, lse, g)
    torch.cuda.synchronize()
    for x, y in zip(bal, again):
        assert torch.equal(x, y)
