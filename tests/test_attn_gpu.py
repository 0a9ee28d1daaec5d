"""Parity of the CUDA path with the fp64 oracle, through the C ABI, on a B200.

Tolerances (stated for this path): bf16 O max |err| <= 2e-2 and mean |err|
<= 2e-3; fp32 LSE |err| <= 1e-3, over every compared element.

* small shapes and the two smallest synthetic workloads: every element;
* the five large workloads, at full size in the launch configuration the
  benchmark times: every element against the oracle run over all rows on
  every host core (the tolerances' max and mean taken over the whole
  workload), plus properties that hold for every row (finite; O inside the
  convex hull of the visible V rows; LSE >= the diagonal logit and >= the
  mean visible logit);
* exact special cases: causal row 0, zero queries, constant V, GQA equal to
  MHA with repeated K/V heads.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    tess.load_library()
    assert tess.tessera_attn_device_error() == 0


def run_gpu(q, k, v, causal=True, scale=None):
    """q, k, v: bf16 CPU tensors. Returns (o fp32 CPU, lse fp32 CPU)."""
    dev = torch.device("cuda:0")
    o, lse = tess.attn_fwd(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    return o.float().cpu(), lse.cpu()


def check(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    lse_gpu = np.asarray(lse_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    lerr = np.abs(lse_gpu - lse_ref)
    assert np.all(np.isfinite(o_gpu)) and np.all(np.isfinite(lse_gpu)), what
    assert err.max() <= MAX_ABS, f"{what}: O max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: O mean abs err {err.mean():.3e}"
    assert lerr.max() <= LSE_ABS, f"{what}: LSE max abs err {lerr.max():.3e}"
    return float(err.max()), float(err.mean()), float(lerr.max())


def check_whole(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """check() over a whole large workload, one (b, h) plane at a time so the
    fp64 temporaries stay small; the max and mean are the whole tensor's."""
    B, Hq = o_ref.shape[:2]
    emax = esum = lmax = 0.0
    for b in range(B):
        for h in range(Hq):
            og = o_gpu[b, h].astype(np.float64)
            assert np.all(np.isfinite(og)) and np.all(np.isfinite(lse_gpu[b, h])), what
            e = np.abs(og - o_ref[b, h])
            emax = max(emax, float(e.max()))
            esum += float(e.sum())
            lmax = max(lmax, float(np.abs(lse_gpu[b, h].astype(np.float64) - lse_ref[b, h]).max()))
    emean = esum / o_ref.size
    assert emax <= MAX_ABS, f"{what}: O max abs err {emax:.3e}"
    assert emean <= MEAN_ABS, f"{what}: O mean abs err {emean:.3e}"
    assert lmax <= LSE_ABS, f"{what}: LSE max abs err {lmax:.3e}"
    return emax, emean, lmax


def oracle_full(q, k, v, causal, scale):
    return oracle.attn_fwd_f64(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                               causal=causal, scale=scale)


# (B, Hq, Hkv, T, d, causal): tails, single tiles, G odd / even / 1, non-causal
SMALL = [
    (1, 2, 1, 1, 64, True), (1, 2, 1, 2, 128, True), (2, 4, 2, 63, 64, True),
    (1, 2, 2, 127, 128, True), (1, 4, 1, 128, 64, True), (2, 2, 1, 129, 128, True),
    (1, 3, 1, 255, 64, True), (1, 3, 3, 256, 128, True), (1, 6, 2, 300, 64, True),
    (1, 8, 1, 385, 128, True), (1, 1, 1, 640, 64, True), (2, 6, 3, 200, 128, True),
    (1, 2, 1, 1, 64, False), (1, 4, 2, 100, 64, False), (1, 3, 1, 129, 128, False),
    (2, 2, 2, 256, 128, False), (1, 4, 4, 383, 64, False), (1, 8, 2, 520, 128, False),
    # more head-dimension-128 shapes: an odd number of 128-row blocks with G
    # odd (a unit's second tile lies past T), key tails of at most 64 rows,
    # units of one, two and many key tiles
    (1, 3, 1, 300, 128, True), (1, 1, 1, 640, 128, True), (1, 5, 5, 333, 128, False),
    (2, 4, 1, 1000, 128, True), (1, 2, 1, 64, 128, True), (3, 6, 2, 190, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,T,d,causal", SMALL)
def test_small_shapes_every_element(B, Hq, Hkv, T, d, causal):
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=1000 + T + d, sigma_qk=1.5)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_gpu(q, k, v, causal, scale)
    ro, rlse = oracle_full(q, k, v, causal, scale)
    check(o.numpy(), lse.numpy(), ro, rlse, f"{(B, Hq, Hkv, T, d, causal)}")


@pytest.mark.parametrize("name", [inputs.SMALL, inputs.TAIL])
def test_small_workloads_every_element(name):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    o, lse = run_gpu(q, k, v, True, w.scale)
    ro, rlse = oracle_full(q, k, v, True, w.scale)
    check(o.numpy(), lse.numpy(), ro, rlse, name)


LARGE = [n for n in inputs.WORKLOADS if n not in (inputs.SMALL, inputs.TAIL)]


def _row_properties(q, k, v, o, lse, scale, G):
    """Checks that hold for every output row, computed on the GPU in fp32."""
    dev = torch.device("cuda:0")
    qf, kf, vf = q.to(dev).float(), k.to(dev).float(), v.to(dev).float()
    kf = kf.repeat_interleave(G, dim=1)
    vf = vf.repeat_interleave(G, dim=1)
    of, lf = o.to(dev), lse.to(dev)
    assert torch.isfinite(of).all() and torch.isfinite(lf).all()
    # O is a convex combination of the visible V rows (bf16 rounding slack)
    lo = torch.cummin(vf, dim=2).values
    hi = torch.cummax(vf, dim=2).values
    slack = 1e-2 * torch.maximum(lo.abs(), hi.abs()) + 1e-6
    assert (of >= lo - slack).all() and (of <= hi + slack).all()
    # LSE >= the diagonal logit, and >= the mean visible logit (Jensen)
    diag = scale * (qf * kf).sum(-1)
    assert (lf >= diag - 1e-3 - 1e-5 * diag.abs()).all()
    T = q.shape[2]
    kmean = torch.cumsum(kf.double(), dim=2) / torch.arange(1, T + 1, device=dev,
                                                            dtype=torch.float64)[:, None]
    jensen = scale * (qf.double() * kmean).sum(-1)
    assert (lf.double() >= jensen - 1e-3 - 1e-5 * jensen.abs()).all()


@pytest.mark.parametrize("name", LARGE)
def test_large_workloads_every_element(name, parity_log):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    o, lse = run_gpu(q, k, v, True, w.scale)
    import time
    t0 = time.perf_counter()
    ro, rlse = oracle.attn_fwd_bf16_threaded(inputs.bf16_bits(q), inputs.bf16_bits(k),
                                             inputs.bf16_bits(v), causal=True, scale=w.scale)
    el = time.perf_counter() - t0
    emax, emean, lmax = check_whole(o.numpy(), lse.numpy(), ro, rlse, name)
    parity_log(test="forward every element", workload=name, o_max_abs=emax, o_mean_abs=emean,
               lse_max_abs=lmax, elements=int(ro.size), oracle_s=round(el, 1),
               oracle_threads=oracle.host_threads())
    _row_properties(q, k, v, o, lse, w.scale, w.G)


def test_long_sequence_beyond_the_largest_workload():
    B, Hq, Hkv, T, d = 1, 2, 1, 32768 + 77, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=99, sigma_qk=2.0)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_gpu(q, k, v, True, scale)
    rows = inputs.sample_rows(B, Hq, T, 24, seed=5)
    ro, rlse = oracle.attn_rows_bf16(inputs.bf16_bits(q), inputs.bf16_bits(k),
                                     inputs.bf16_bits(v), rows, causal=True, scale=scale)
    b, h, i = rows.T
    check(o[b, h, i].numpy(), lse[b, h, i].numpy(), ro, rlse, "T=32845")


@pytest.mark.parametrize("d", [64, 128])
def test_causal_row_zero_is_exact(d):
    B, Hq, Hkv, T = 2, 8, 2, 300
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=3, sigma_qk=4.0)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_gpu(q, k, v, True, scale)
    vrep = v.float().repeat_interleave(Hq // Hkv, dim=1)
    assert torch.equal(o[:, :, 0], vrep[:, :, 0])  # p = 1, l = 1: bit exact
    s00 = scale * (q.double()[:, :, 0] * k.double().repeat_interleave(4, 1)[:, :, 0]).sum(-1)
    assert torch.allclose(lse[:, :, 0].double(), s00, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("causal", [True, False])
def test_zero_queries_give_prefix_means(causal):
    B, Hq, Hkv, T, d = 1, 4, 2, 333, 64
    _, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=4)
    q = torch.zeros((B, Hq, T, d), dtype=torch.bfloat16)
    o, lse = run_gpu(q, k, v, causal, 0.125)
    vd = v.double().repeat_interleave(2, dim=1)
    n = torch.arange(1, T + 1, dtype=torch.float64)
    want = torch.cumsum(vd, 2) / n[:, None] if causal else vd.mean(2, keepdim=True).expand_as(vd)
    want_lse = torch.log(n) if causal else torch.full((T,), math.log(T), dtype=torch.float64)
    check(o.numpy(), lse.numpy(), want.numpy(), want_lse.expand(B, Hq, T).numpy(), "Q=0")


def test_constant_and_unit_values():
    B, Hq, Hkv, T, d = 2, 4, 1, 260, 128
    q, k, _ = inputs.make_qkv(B, Hq, Hkv, T, d, seed=6, sigma_qk=3.0)
    c = torch.linspace(-3, 3, d).to(torch.bfloat16)
    v = c.expand(B, Hkv, T, d).contiguous()
    o, _ = run_gpu(q, k, v, True, 1.0 / math.sqrt(d))
    # P is rounded to bf16, so O = c * (sum of rounded p) / l: within 2^-8 relative
    assert torch.allclose(o, c.float().expand_as(o), rtol=2 ** -7, atol=1e-6)
    ones = torch.ones((B, Hkv, T, d), dtype=torch.bfloat16)
    o1, _ = run_gpu(q, k, ones, True, 1.0 / math.sqrt(d))
    assert torch.allclose(o1, torch.ones_like(o1), rtol=0, atol=2 ** -7)


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (6, 3), (4, 1)])
def test_gqa_equals_mha_with_repeated_heads(Hq, Hkv):
    B, T, d = 2, 410, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=8)
    G = Hq // Hkv
    o, lse = run_gpu(q, k, v, True, 0.1)
    om, lsem = run_gpu(q, k.repeat_interleave(G, 1).contiguous(),
                       v.repeat_interleave(G, 1).contiguous(), True, 0.1)
    # per-tile arithmetic does not depend on how tiles are paired in a CTA
    assert torch.equal(o, om) and torch.equal(lse, lsem)


def test_outputs_do_not_spill_past_their_buffers():
    B, Hq, Hkv, T, d = 1, 4, 2, 200, 64
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=9)
    dev = torch.device("cuda:0")
    guard = 4096
    n_o = B * Hq * T * d
    n_l = B * Hq * T
    obuf = torch.full((n_o + 2 * guard,), 7.0, dtype=torch.bfloat16, device=dev)
    lbuf = torch.full((n_l + 2 * guard,), -7.0, dtype=torch.float32, device=dev)
    o = obuf[guard:guard + n_o].view(B, Hq, T, d)
    lse = lbuf[guard:guard + n_l].view(B, Hq, T)
    tess.attn_fwd(q.to(dev), k.to(dev), v.to(dev), out=o, lse=lse)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    assert (obuf[:guard] == 7.0).all() and (obuf[guard + n_o:] == 7.0).all()
    assert (lbuf[:guard] == -7.0).all() and (lbuf[guard + n_l:] == -7.0).all()
    ro, rlse = oracle_full(q, k, v, True, 1.0 / math.sqrt(d))
    check(o.float().cpu().numpy(), lse.cpu().numpy(), ro, rlse, "guarded")


def test_lse_may_be_omitted_and_results_repeat_bitwise():
    B, Hq, Hkv, T, d = 1, 8, 2, 700, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=10)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o1, l1 = tess.attn_fwd(qd, kd, vd)
    o2, l2 = tess.attn_fwd(qd, kd, vd, want_lse=False)
    assert l2 is None
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o3, l3 = tess.attn_fwd(qd, kd, vd)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(o1, o3) and torch.equal(l1, l3)


@pytest.mark.parametrize("B,Hq,Hkv,T,d", [(8, 32, 32, 2048, 128), (8, 16, 8, 8192, 128),
                                          (8, 8, 4, 32768, 64)])
def test_l2_grouped_unit_order_matches_per_batch_calls_bitwise(B, Hq, Hkv, T, d):
    # K/V larger than L2, so the units walk groups of (batch, K/V head) slices;
    # one batch alone fits and keeps the global order.  Units never share
    # arithmetic, so the order must not change a bit.
    dev = torch.device("cuda:0")
    kv_bytes = 2 * B * Hkv * T * d * 2
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    assert kv_bytes > l2 and kv_bytes // B <= l2
    g = torch.Generator(device=dev)
    g.manual_seed(31)
    q, k, v = (torch.randn((B, h, T, d), generator=g, device=dev).to(torch.bfloat16)
               for h in (Hq, Hkv, Hkv))
    o, lse = tess.attn_fwd(q, k, v)
    for b in range(B):
        ob, lb = tess.attn_fwd(q[b:b + 1], k[b:b + 1], v[b:b + 1])
        assert torch.equal(ob, o[b:b + 1]) and torch.equal(lb, lse[b:b + 1]), b
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0


def test_empty_inputs_launch_nothing():
    dev = torch.device("cuda:0")
    q = torch.empty((0, 4, 16, 64), dtype=torch.bfloat16, device=dev)
    k = torch.empty((0, 2, 16, 64), dtype=torch.bfloat16, device=dev)
    o, lse = tess.attn_fwd(q, k, k)
    assert o.numel() == 0 and tess.tessera_attn_last_launch_count() == 0
    q = torch.empty((1, 4, 0, 64), dtype=torch.bfloat16, device=dev)
    k = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=dev)
    o, lse = tess.attn_fwd(q, k, k)
    assert o.numel() == 0 and tess.tessera_attn_last_launch_count() == 0


def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    import time
    assert tess.tessera_attn_device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    assert tess.tessera_attn_selftest_timeout(50_000, stream) == 0  # 50 ms limit
    t0 = time.time()
    code = tess.tessera_attn_device_error()
    assert code == tess.DEVICE_ERR_SELFTEST
    assert time.time() - t0 < 5.0
    assert tess.tessera_attn_device_error() == 0  # read clears the word
    # the context still works: a normal call afterwards is correct
    B, Hq, Hkv, T, d = 1, 4, 2, 200, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=11)
    o, lse = run_gpu(q, k, v, True, 1.0 / math.sqrt(d))
    ro, rlse = oracle_full(q, k, v, True, 1.0 / math.sqrt(d))
    check(o.numpy(), lse.numpy(), ro, rlse, "after self-test")


@pytest.mark.parametrize("B,Hq,Hkv,T,d,causal,chunks", [
    (1, 32, 8, 1000, 128, True, 0), (2, 6, 3, 129, 64, True, 4), (3, 4, 2, 77, 128, True, 1),
    (2, 8, 2, 300, 64, False, 100), (1, 2, 1, 1, 64, True, 0),
    (2, 6, 1, 129, 64, True, 7), (1, 8, 2, 300, 128, False, 5), (4, 4, 4, 200, 128, True, 0),
])
def test_host_pipeline_matches_device_call_bitwise(B, Hq, Hkv, T, d, causal, chunks):
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=21 + T, sigma_qk=2.0)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = run_gpu(q, k, v, causal, scale)
    qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o_h, lse_h = tess.attn_fwd_host(qp, kp, vp, causal=causal, scale=scale, chunks=chunks)
    assert tess.tessera_attn_last_launch_count() == len(tess.tessera_attn_fwd_host_plan(B, Hq, Hkv, chunks))
    assert tess.tessera_attn_device_error() == 0
    assert torch.equal(o_h.float(), o_ref) and torch.equal(lse_h, lse_ref)


def test_host_pipeline_pageable_inputs_and_no_lse():
    B, Hq, Hkv, T, d = 2, 4, 2, 260, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=5)
    o_ref, _ = run_gpu(q, k, v, True, 0.1)
    o_h, lse_h = tess.attn_fwd_host(q, k, v, causal=True, scale=0.1, want_lse=False)
    assert lse_h is None
    assert torch.equal(o_h.float(), o_ref)


@pytest.mark.parametrize("causal", [True, False])
def test_running_max_rescale_path(causal):
    # Logits that grow by ~144 (log2 units) per key tile, so the running max
    # moves past the lazy-rescale threshold (64) in every tile and O is rescaled.
    B, Hq, Hkv, T, d = 1, 4, 2, 640, 128
    _, _, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=17)
    q = torch.ones((B, Hq, T, d), dtype=torch.bfloat16)
    ramp = (torch.arange(T, dtype=torch.float32) * (100.0 / 128.0) / math.sqrt(d))
    k = ramp[None, None, :, None].expand(B, Hkv, T, d).to(torch.bfloat16).contiguous()
    scale = 1.0 / math.sqrt(d)
    o, lse = run_gpu(q, k, v, causal, scale)
    ro, rlse = oracle_full(q, k, v, causal, scale)
    check(o.numpy(), lse.numpy(), ro, rlse, f"rescale causal={causal}")


@pytest.mark.parametrize("log2_big", [20, 40])
def test_large_values_stay_finite(log2_big):
    # V far from unit scale with peaky softmax rows (Q/K sigma 4): O scales with
    # V.  2^40 * T * the 2^64 weight bound of the lazy rescale stays below 2^128.
    B, Hq, Hkv, T, d = 1, 4, 1, 2048, 128
    q, k, v = inputs.make_qkv(B, Hq, Hkv, T, d, seed=23, sigma_qk=4.0)
    big = 2.0 ** log2_big
    vb = (v.float() * big).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_gpu(q, k, vb, True, scale)
    rows = inputs.sample_rows(B, Hq, T, 64, seed=3)
    ro, rlse = oracle.attn_rows_bf16(inputs.bf16_bits(q), inputs.bf16_bits(k), inputs.bf16_bits(vb),
                                     rows, causal=True, scale=scale)
    b, h, i = rows.T
    check(o[b, h, i].numpy() / big, lse[b, h, i].numpy(), ro / big, rlse, f"V * 2^{log2_big}")
