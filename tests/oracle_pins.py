"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes a loaded oracle library (the real one, or one
built from a copy of the source with a planted mistake) and raises
AssertionError when the oracle disagrees with what the mathematics fixes:

* hand-derived closed forms (tests/golden/closed_forms.yaml);
* a library routine: torch's CPU scaled_dot_product_attention in float64,
  with K/V heads repeated for grouped-query attention, and torch.logsumexp
  for the LSE;
* exact arithmetic: Python Decimal at 60 significant digits on tiny inputs
  whose logits are far beyond exp's fp64 range;
* invariants: causal row 0, identical V rows, uniform weights for zero
  queries (prefix means, LSE = ln(i+1)), GQA == MHA with repeated K/V,
  invariance to a common shift of every key, joint key/value permutation,
  scale homogeneity, convexity of O.
"""
from __future__ import annotations

import math
import os
from decimal import Decimal, getcontext

import numpy as np
import torch
import yaml

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "closed_forms.yaml")

_MATH_NAMES = {"sqrt": math.sqrt, "log": math.log, "exp": math.exp}


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, _MATH_NAMES))


def _rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).normal(0.0, sigma, size=shape)


def pin_closed_forms(lib):
    with open(GOLDEN) as f:
        cases = yaml.safe_load(f)
    for name, c in cases.items():
        B, Hq, Hkv, T, d = c["B"], c["Hq"], c["Hkv"], c["T"], c["d"]
        q = np.array([_eval(x) for x in c["q"]]).reshape(B, Hq, T, d)
        k = np.array([_eval(x) for x in c["k"]]).reshape(B, Hkv, T, d)
        v = np.array([_eval(x) for x in c["v"]]).reshape(B, Hkv, T, d)
        scale = _eval(c["scale"])
        for mode, causal in (("causal", True), ("full", False)):
            o, lse = oracle.attn_fwd_f64(q, k, v, causal=causal, scale=scale, lib=lib)
            want_o = np.array([_eval(x) for x in c[mode]["o"]]).reshape(o.shape)
            want_lse = np.array([_eval(x) for x in c[mode]["lse"]]).reshape(lse.shape)
            assert np.allclose(o, want_o, rtol=0, atol=1e-14), (name, mode, o, want_o)
            assert np.allclose(lse, want_lse, rtol=0, atol=1e-14), (name, mode, lse, want_lse)


def _torch_reference(q, k, v, causal, scale):
    """torch CPU float64 SDPA with K/V heads repeated (repeat_interleave)."""
    G = q.shape[1] // k.shape[1]
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal,
                                                         scale=scale)
    s = scale * (qt @ kt.transpose(-1, -2))
    if causal:
        T = q.shape[2]
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy()


def pin_library_sdpa(lib):
    shapes = [  # (B, Hq, Hkv, T, d, causal, sigma)
        (1, 1, 1, 1, 4, True, 1.0),
        (2, 4, 2, 17, 8, True, 1.0),
        (1, 6, 3, 33, 16, False, 1.0),
        (2, 8, 2, 40, 64, True, 4.0),
        (1, 4, 1, 65, 32, True, 2.0),
        (1, 3, 3, 9, 5, False, 3.0),
    ]
    for n, (B, Hq, Hkv, T, d, causal, sigma) in enumerate(shapes):
        q = _rand((B, Hq, T, d), 10 + n, sigma)
        k = _rand((B, Hkv, T, d), 20 + n, sigma)
        v = _rand((B, Hkv, T, d), 30 + n)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn_fwd_f64(q, k, v, causal=causal, scale=scale, lib=lib)
        ro, rlse = _torch_reference(q, k, v, causal, scale)
        assert np.max(np.abs(o - ro)) <= 1e-12, ("O", n, np.max(np.abs(o - ro)))
        assert np.max(np.abs(lse - rlse)) <= 1e-12, ("LSE", n, np.max(np.abs(lse - rlse)))


def _decimal_attention(q, k, v, causal, scale):
    """Exact-ish attention in Decimal arithmetic (60 digits), one row at a time."""
    getcontext().prec = 60
    B, Hq, T, d = q.shape
    G = Hq // k.shape[1]
    o = np.zeros(q.shape)
    lse = np.zeros(q.shape[:3])
    sc = Decimal(scale)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for i in range(T):
                keys = range(i + 1) if causal else range(T)
                s = [sc * sum(Decimal(float(q[b, h, i, c])) * Decimal(float(k[b, g, j, c]))
                              for c in range(d)) for j in keys]
                e = [x.exp() for x in s]  # Decimal has no overflow at these magnitudes
                z = sum(e)
                for c in range(d):
                    o[b, h, i, c] = float(sum(e[n] * Decimal(float(v[b, g, j, c]))
                                              for n, j in enumerate(keys)) / z)
                lse[b, h, i] = float(z.ln())
    return o, lse


def pin_decimal_large_logits(lib):
    for n, (B, Hq, Hkv, T, d, causal, sigma) in enumerate([
            (1, 2, 1, 5, 3, True, 30.0),     # logits ~ +-1500: exp overflows in fp64
            (1, 2, 2, 4, 2, False, 25.0),
            (1, 4, 2, 3, 4, True, 0.5)]):
        q = _rand((B, Hq, T, d), 40 + n, sigma)
        k = _rand((B, Hkv, T, d), 50 + n, sigma)
        v = _rand((B, Hkv, T, d), 60 + n)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.attn_fwd_f64(q, k, v, causal=causal, scale=scale, lib=lib)
        eo, else_ = _decimal_attention(q, k, v, causal, scale)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse)), ("non-finite", n)
        assert np.max(np.abs(o - eo)) <= 1e-12 * max(1.0, np.max(np.abs(eo))), ("O", n)
        assert np.max(np.abs(lse - else_)) <= 1e-12 * max(1.0, np.max(np.abs(else_))), ("LSE", n)


def pin_invariants(lib):
    B, Hq, Hkv, T, d = 2, 6, 2, 37, 8
    G = Hq // Hkv
    scale = 0.3
    q = _rand((B, Hq, T, d), 1)
    k = _rand((B, Hkv, T, d), 2)
    v = _rand((B, Hkv, T, d), 3)
    o, lse = oracle.attn_fwd_f64(q, k, v, causal=True, scale=scale, lib=lib)

    # causal row 0 attends to key 0 only: O = V[g, 0] exactly, LSE = s_00
    for h in range(Hq):
        g = h // G
        assert np.array_equal(o[:, h, 0], v[:, g, 0]), "causal row 0 != V[0]"
        s00 = scale * np.einsum("bc,bc->b", q[:, h, 0], k[:, g, 0])
        assert np.allclose(lse[:, h, 0], s00, rtol=0, atol=1e-14), "LSE row 0 != s00"

    # identical V rows give that row back
    c = _rand((B, Hkv, 1, d), 4)
    o_c, _ = oracle.attn_fwd_f64(q, k, np.repeat(c, T, axis=2), causal=True, scale=scale, lib=lib)
    assert np.allclose(o_c, np.repeat(np.repeat(c, G, axis=1), T, axis=2), rtol=0, atol=1e-14)

    # zero queries: uniform weights over the visible prefix
    z = np.zeros_like(q)
    o_z, lse_z = oracle.attn_fwd_f64(z, k, v, causal=True, scale=scale, lib=lib)
    prefix_mean = np.cumsum(v, axis=2) / np.arange(1, T + 1)[None, None, :, None]
    assert np.allclose(o_z, np.repeat(prefix_mean, G, axis=1), rtol=0, atol=1e-13)
    assert np.allclose(lse_z, np.log(np.arange(1, T + 1))[None, None, :], rtol=0, atol=1e-14)
    o_zf, lse_zf = oracle.attn_fwd_f64(z, k, v, causal=False, scale=scale, lib=lib)
    assert np.allclose(o_zf, np.repeat(v.mean(axis=2, keepdims=True), Hq // Hkv, axis=1)
                       .repeat(T, axis=2), rtol=0, atol=1e-13)
    assert np.allclose(lse_zf, math.log(T), rtol=0, atol=1e-14)

    # GQA equals MHA with K/V heads repeated, bit for bit
    o_m, lse_m = oracle.attn_fwd_f64(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1),
                                     causal=True, scale=scale, lib=lib)
    assert np.array_equal(o_m, o) and np.array_equal(lse_m, lse), "GQA != repeated MHA"

    # the last causal row sees every key: equal to the non-causal last row
    o_f, lse_f = oracle.attn_fwd_f64(q, k, v, causal=False, scale=scale, lib=lib)
    assert np.array_equal(o_f[:, :, -1], o[:, :, -1]) and np.array_equal(lse_f[:, :, -1], lse[:, :, -1])

    # adding one vector to every key shifts each row's logits by a constant
    shift = _rand((B, Hkv, 1, d), 5)
    o_s, lse_s = oracle.attn_fwd_f64(q, k + shift, v, causal=True, scale=scale, lib=lib)
    delta = scale * np.einsum("bhtc,bhc->bht", q, np.repeat(shift[:, :, 0], G, axis=1))
    assert np.allclose(o_s, o, rtol=0, atol=1e-12), "O not shift invariant"
    assert np.allclose(lse_s, lse + delta, rtol=0, atol=1e-12), "LSE shift wrong"

    # permuting keys and values together leaves non-causal attention unchanged
    perm = np.random.default_rng(6).permutation(T)
    o_p, lse_p = oracle.attn_fwd_f64(q, k[:, :, perm], v[:, :, perm], causal=False,
                                     scale=scale, lib=lib)
    assert np.allclose(o_p, o_f, rtol=0, atol=1e-13) and np.allclose(lse_p, lse_f, rtol=0, atol=1e-13)

    # scale is a plain multiplier of the logits
    o_h, lse_h = oracle.attn_fwd_f64(2.0 * q, k, v, causal=True, scale=scale / 2.0, lib=lib)
    assert np.allclose(o_h, o, rtol=0, atol=1e-13) and np.allclose(lse_h, lse, rtol=0, atol=1e-13)

    # O is a convex combination of the visible V rows
    for h in range(Hq):
        g = h // G
        lo = np.minimum.accumulate(v[:, g], axis=1)
        hi = np.maximum.accumulate(v[:, g], axis=1)
        assert np.all(o[:, h] >= lo - 1e-13) and np.all(o[:, h] <= hi + 1e-13)


def pin_rows_entry(lib):
    """The bf16 row entry agrees bit for bit with the full fp64 entry."""
    from causal_gqa_attention_03_b200.inputs import make_qkv, bf16_bits, sample_rows
    B, Hq, Hkv, T, d = 2, 4, 2, 150, 64
    q, k, v = make_qkv(B, Hq, Hkv, T, d, seed=7, sigma_qk=2.0)
    scale = 1.0 / 8.0
    for causal in (True, False):
        o, lse = oracle.attn_fwd_f64(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                     causal=causal, scale=scale, lib=lib)
        rows = sample_rows(B, Hq, T, 64, seed=8)
        ro, rlse = oracle.attn_rows_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v), rows,
                                         causal=causal, scale=scale, lib=lib)
        b, h, i = rows.T
        assert np.array_equal(ro, o[b, h, i]) and np.array_equal(rlse, lse[b, h, i])


# ------------------------------------------------------------------ backward
def _torch_grads(q, k, v, dout, causal, scale):
    """torch CPU float64 autograd of SDPA with K/V heads repeated; the gradients
    of the repeated heads are summed back onto each K/V head by autograd."""
    G = q.shape[1] // k.shape[1]
    qt = torch.tensor(q, requires_grad=True)
    kt = torch.tensor(k, requires_grad=True)
    vt = torch.tensor(v, requires_grad=True)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1), is_causal=causal,
        scale=scale)
    o.backward(torch.from_numpy(dout))
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def pin_bwd_library_autograd(lib):
    shapes = [  # (B, Hq, Hkv, T, d, causal, sigma)
        (1, 1, 1, 1, 4, True, 1.0),
        (2, 4, 2, 17, 8, True, 1.0),
        (1, 6, 3, 33, 16, False, 1.0),
        (2, 8, 2, 40, 32, True, 3.0),
        (1, 4, 1, 29, 8, False, 2.0),
    ]
    for n, (B, Hq, Hkv, T, d, causal, sigma) in enumerate(shapes):
        q = _rand((B, Hq, T, d), 40 + n, sigma)
        k = _rand((B, Hkv, T, d), 50 + n, sigma)
        v = _rand((B, Hkv, T, d), 60 + n)
        g = _rand((B, Hq, T, d), 70 + n)
        scale = 1.0 / math.sqrt(d)
        dq, dk, dv = oracle.attn_bwd_f64(q, k, v, g, causal=causal, scale=scale, lib=lib)
        rq, rk, rv = _torch_grads(q, k, v, g, causal, scale)
        for name, a, r in (("dQ", dq, rq), ("dK", dk, rk), ("dV", dv, rv)):
            err = np.max(np.abs(a - r)) / max(1.0, np.max(np.abs(r)))
            assert err <= 1e-12, (name, n, err)


def pin_bwd_finite_differences(lib):
    """Central differences of L = sum(O * dO), O from the forward entry."""
    B, Hq, Hkv, T, d = 1, 2, 1, 5, 3
    scale = 0.7
    q = _rand((B, Hq, T, d), 81)
    k = _rand((B, Hkv, T, d), 82)
    v = _rand((B, Hkv, T, d), 83)
    g = _rand((B, Hq, T, d), 84)
    eps = 1e-5
    for causal in (True, False):
        grads = oracle.attn_bwd_f64(q, k, v, g, causal=causal, scale=scale, lib=lib)
        for which, x in enumerate((q, k, v)):
            for idx in np.ndindex(x.shape):
                xs = [q.copy(), k.copy(), v.copy()]
                xs[which][idx] += eps
                lp = np.sum(oracle.attn_fwd_f64(*xs, causal=causal, scale=scale, lib=lib)[0] * g)
                xs[which][idx] -= 2 * eps
                lm = np.sum(oracle.attn_fwd_f64(*xs, causal=causal, scale=scale, lib=lib)[0] * g)
                fd = (lp - lm) / (2 * eps)
                assert abs(fd - grads[which][idx]) <= 1e-8, (causal, which, idx, fd,
                                                             grads[which][idx])


def pin_bwd_invariants(lib):
    B, Hq, Hkv, T, d = 2, 6, 2, 23, 8
    G = Hq // Hkv
    scale = 0.4
    q = _rand((B, Hq, T, d), 91, 2.0)
    k = _rand((B, Hkv, T, d), 92, 2.0)
    v = _rand((B, Hkv, T, d), 93)
    g = _rand((B, Hq, T, d), 94)
    for causal in (True, False):
        dq, dk, dv = oracle.attn_bwd_f64(q, k, v, g, causal=causal, scale=scale, lib=lib)
        # rows of P sum to one: the keys' dV add up to the group's dO
        want = g.reshape(B, Hkv, G, T, d).sum(axis=(2, 3))
        assert np.allclose(dv.sum(axis=2), want, rtol=0, atol=1e-12), "sum_j dV != sum dO"
        # rows of dS sum to zero: the keys' dK add up to zero
        assert np.allclose(dk.sum(axis=2), 0.0, rtol=0, atol=1e-12), "sum_j dK != 0"
        # GQA equals MHA with repeated K/V heads, the repeats' gradients summed
        mq, mk, mv = oracle.attn_bwd_f64(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), g,
                                         causal=causal, scale=scale, lib=lib)
        assert np.array_equal(mq, dq), "GQA dQ != repeated-MHA dQ"
        assert np.allclose(mk.reshape(B, Hkv, G, T, d).sum(axis=2), dk, rtol=0, atol=1e-13)
        assert np.allclose(mv.reshape(B, Hkv, G, T, d).sum(axis=2), dv, rtol=0, atol=1e-13)
        # dS does not depend on how the scale is split between q and scale
        hq, _, _ = oracle.attn_bwd_f64(2.0 * q, k, v, g, causal=causal, scale=scale / 2.0,
                                       lib=lib)
        assert np.allclose(hq, dq / 2.0, rtol=0, atol=1e-13), "dQ scale split"
        # zero upstream gradient
        zq, zk, zv = oracle.attn_bwd_f64(q, k, v, np.zeros_like(g), causal=causal,
                                         scale=scale, lib=lib)
        assert not zq.any() and not zk.any() and not zv.any()
    # one key: P = 1, so dS = 0 and dV is the group's dO
    q1, k1, v1, g1 = q[:, :, :1], k[:, :, :1], v[:, :, :1], g[:, :, :1]
    dq, dk, dv = oracle.attn_bwd_f64(q1, k1, v1, g1, causal=True, scale=scale, lib=lib)
    assert np.allclose(dq, 0.0, rtol=0, atol=1e-15) and np.allclose(dk, 0.0, rtol=0, atol=1e-15)
    assert np.allclose(dv, g1.reshape(B, Hkv, G, 1, d).sum(axis=2), rtol=0, atol=1e-15)


def pin_bwd_dq_rows_entry(lib):
    """The bf16 dQ-row entry agrees bit for bit with the full fp64 backward."""
    from causal_gqa_attention_03_b200.inputs import make_qkv, bf16_bits, sample_rows
    B, Hq, Hkv, T, d = 1, 4, 2, 70, 16
    q, k, v = make_qkv(B, Hq, Hkv, T, d, seed=11, sigma_qk=2.0)
    gq, _, _ = make_qkv(B, Hq, Hkv, T, d, seed=12)
    scale = 0.25
    for causal in (True, False):
        dq, _, _ = oracle.attn_bwd_f64(q.double().numpy(), k.double().numpy(),
                                       v.double().numpy(), gq.double().numpy(),
                                       causal=causal, scale=scale, lib=lib)
        rows = sample_rows(B, Hq, T, 40, seed=13)
        rq = oracle.attn_bwd_dq_rows_bf16(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                          bf16_bits(gq), rows, causal=causal, scale=scale,
                                          lib=lib)
        b, h, i = rows.T
        assert np.array_equal(rq, dq[b, h, i])


# ------------------------------------------------------------- paged decode
def _gathered(k_cache, tab, b, n):
    bs = k_cache.shape[2]
    return np.stack([k_cache[tab[b, j // bs], :, j % bs] for j in range(n)], axis=1)  # [Hkv,n,d]


def _paged_case(seed, B, Hq, Hkv, d, bs, lens, sigma=1.0):
    from causal_gqa_attention_03_b200.inputs import make_paged
    q, k, v, tab, lens = make_paged(B, Hq, Hkv, d, bs, lens, seed=seed, sigma_qk=sigma)
    return q.double().numpy(), k.double().numpy(), v.double().numpy(), tab, lens


def pin_decode_library(lib):
    cases = [  # (B, Hq, Hkv, d, bs, lens, sigma)
        (3, 8, 2, 16, 4, [1, 9, 17], 1.0),
        (2, 4, 4, 8, 1, [5, 3], 2.0),
        (2, 6, 1, 32, 16, [40, 16], 3.0),
    ]
    for n_case, (B, Hq, Hkv, d, bs, lens, sigma) in enumerate(cases):
        q, k, v, tab, lens = _paged_case(100 + n_case, B, Hq, Hkv, d, bs, lens, sigma)
        scale = 1.0 / math.sqrt(d)
        o, lse = oracle.paged_decode_f64(q, k, v, tab, lens, scale=scale, lib=lib)
        G = Hq // Hkv
        for b in range(B):
            n = int(lens[b])
            kk = torch.from_numpy(_gathered(k, tab, b, n)).repeat_interleave(G, dim=0)
            vv = torch.from_numpy(_gathered(v, tab, b, n)).repeat_interleave(G, dim=0)
            qq = torch.from_numpy(q[b])[:, None, :]
            ro = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)
            rl = torch.logsumexp(scale * (qq @ kk.transpose(-1, -2)), dim=-1)
            assert np.max(np.abs(o[b] - ro[:, 0].numpy())) <= 1e-12, (n_case, b)
            assert np.max(np.abs(lse[b] - rl[:, 0].numpy())) <= 1e-12, (n_case, b)


def pin_decode_invariants(lib):
    B, Hq, Hkv, d, bs = 3, 8, 2, 16, 4
    q, k, v, tab, lens = _paged_case(7, B, Hq, Hkv, d, bs, [6, 1, 13])
    scale = 0.3
    o, lse = oracle.paged_decode_f64(q, k, v, tab, lens, scale=scale, lib=lib)
    # moving the physical blocks (and the table with them) changes nothing
    perm = np.random.default_rng(3).permutation(k.shape[0])
    inv = np.argsort(perm)
    k2, v2 = k[perm], v[perm]
    tab2 = np.where(tab >= 0, inv[np.maximum(tab, 0)], -1).astype(np.int32)
    o2, lse2 = oracle.paged_decode_f64(q, k2, v2, tab2, lens, scale=scale, lib=lib)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2), "block placement"
    # re-paging the same tokens with blocks of one token changes nothing
    n_tok = int(lens.sum())
    k1 = np.zeros((n_tok, Hkv, 1, d)); v1 = np.zeros((n_tok, Hkv, 1, d))
    tab1 = np.full((B, int(lens.max())), -1, dtype=np.int32)
    pos = 0
    for b in range(B):
        for j in range(int(lens[b])):
            k1[pos, :, 0] = k[tab[b, j // bs], :, j % bs]
            v1[pos, :, 0] = v[tab[b, j // bs], :, j % bs]
            tab1[b, j] = pos
            pos += 1
    o1, lse1 = oracle.paged_decode_f64(q, k1, v1, tab1, lens, scale=scale, lib=lib)
    assert np.array_equal(o, o1) and np.array_equal(lse, lse1), "block size"
    # one token: the value row itself, LSE = its logit
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        k0 = k[tab[1, 0], g, 0]; v0 = v[tab[1, 0], g, 0]
        assert np.array_equal(o[1, h], v0)
        assert abs(lse[1, h] - scale * np.dot(q[1, h], k0)) <= 1e-14
    # no tokens: zero output, LSE -inf
    o0, lse0 = oracle.paged_decode_f64(q, k, v, tab, np.array([0, 1, 13], np.int32),
                                       scale=scale, lib=lib)
    assert not o0[0].any() and np.all(np.isneginf(lse0[0]))
    # the decode step equals the last row of a causal forward over the tokens
    for b in range(B):
        n = int(lens[b])
        kk = _gathered(k, tab, b, n)[None]
        vv = _gathered(v, tab, b, n)[None]
        qq = np.zeros((1, Hq, n, d)); qq[0, :, n - 1] = q[b]
        fo, fl = oracle.attn_fwd_f64(qq, kk, vv, causal=True, scale=scale, lib=lib)
        assert np.array_equal(fo[0, :, n - 1], o[b]) and np.array_equal(fl[0, :, n - 1], lse[b])


# ---------------------------------------------------------------- prologue
def pin_rmsnorm_library(lib):
    """torch's RMSNorm (float64) on random rows and weights, eps large enough
    to matter."""
    for seed, (rows, dim, eps, sigma) in enumerate([(5, 64, 1e-6, 1.0), (3, 128, 1e-2, 0.05),
                                                     (4, 4096, 1e-5, 2.0), (2, 7, 0.5, 0.3)]):
        x = _rand((rows, dim), 900 + seed, sigma)
        w = _rand((dim,), 950 + seed)
        got = oracle.rmsnorm_f64(x, w, eps, lib=lib)
        want = torch.nn.functional.rms_norm(torch.from_numpy(x), (dim,),
                                            weight=torch.from_numpy(w), eps=eps).numpy()
        assert np.allclose(got, want, rtol=1e-13, atol=1e-15), (rows, dim, eps)


def pin_rmsnorm_invariants(lib):
    x = _rand((6, 32), 960)
    w = _rand((32,), 961)
    y = oracle.rmsnorm_f64(x, w, 0.0, lib=lib)
    # scale invariance and oddness (eps = 0)
    assert np.allclose(oracle.rmsnorm_f64(3.7 * x, w, 0.0, lib=lib), y, rtol=1e-13, atol=0)
    assert np.array_equal(oracle.rmsnorm_f64(-x, w, 0.0, lib=lib), -y)
    # unit root-mean-square before the weight
    ones = oracle.rmsnorm_f64(x, np.ones(32), 0.0, lib=lib)
    assert np.allclose(np.mean(ones ** 2, axis=1), 1.0, rtol=1e-13)
    # a constant row c gives sign(c) * w
    c = np.full((2, 32), -2.5)
    assert np.allclose(oracle.rmsnorm_f64(c, w, 0.0, lib=lib), -np.tile(w, (2, 1)),
                       rtol=1e-15, atol=1e-15)
    # eps: a row of ones over eps = 3 gives 1 / sqrt(1 + 3) = 0.5 times w
    assert np.allclose(oracle.rmsnorm_f64(np.ones((1, 32)), w, 3.0, lib=lib), 0.5 * w,
                       rtol=1e-15, atol=0)


def _rope_complex(x, pos, base):
    """Rotary embedding as complex multiplication: z_i = x_i + j x_{i+d/2}
    times exp(j p theta_i), theta_i = exp(-ln(base) 2i/d)."""
    d = x.shape[-1]
    half = d // 2
    theta = np.exp(-np.log(base) * 2.0 * np.arange(half) / d)
    z = x[..., :half] + 1j * x[..., half:]
    r = z * np.exp(1j * pos[..., None] * theta)
    return np.concatenate([r.real, r.imag], axis=-1)


def pin_rope_complex(lib):
    for seed, (B, T, Hq, Hkv, d, base, big) in enumerate([(2, 5, 4, 2, 8, 10000.0, False),
                                                           (1, 7, 2, 1, 128, 10000.0, True),
                                                           (2, 3, 3, 3, 64, 500000.0, True)]):
        H3 = Hq + 2 * Hkv
        qkv = _rand((B, T, H3 * d), 970 + seed)
        pos = None
        p = np.tile(np.arange(T, dtype=np.float64), (B, 1))
        if big:
            pos = np.random.default_rng(980 + seed).integers(0, 200000, size=(B, T)).astype(np.int32)
            p = pos.astype(np.float64)
        q, k, v = oracle.rope_qkv_f64(qkv, Hq, Hkv, positions=pos, base=base, lib=lib)
        heads = qkv.reshape(B, T, H3, d)
        want_q = _rope_complex(heads[:, :, :Hq], p[:, :, None], base).transpose(0, 2, 1, 3)
        want_k = _rope_complex(heads[:, :, Hq:Hq + Hkv], p[:, :, None], base).transpose(0, 2, 1, 3)
        # angles up to 2e5 rad: the two routes differ by the rounding of a * theta
        tol = 1e-9 if big else 1e-13
        assert np.allclose(q, want_q, rtol=0, atol=tol), (seed, np.abs(q - want_q).max())
        assert np.allclose(k, want_k, rtol=0, atol=tol), (seed, np.abs(k - want_k).max())
        assert np.array_equal(v, heads[:, :, Hq + Hkv:].transpose(0, 2, 1, 3))


def pin_rope_invariants(lib):
    B, T, Hq, Hkv, d = 2, 6, 2, 1, 16
    qkv = _rand((B, T, (Hq + 2 * Hkv) * d), 990)
    heads = qkv.reshape(B, T, Hq + 2 * Hkv, d)
    # position 0 everywhere: the identity, exactly
    q0, k0, _ = oracle.rope_qkv_f64(qkv, Hq, Hkv, positions=np.zeros((B, T), np.int32), lib=lib)
    assert np.array_equal(q0, heads[:, :, :Hq].transpose(0, 2, 1, 3))
    assert np.array_equal(k0, heads[:, :, Hq:Hq + Hkv].transpose(0, 2, 1, 3))
    # no positions means p = t
    q1, k1, v1 = oracle.rope_qkv_f64(qkv, Hq, Hkv, lib=lib)
    pt = np.tile(np.arange(T, dtype=np.int32), (B, 1))
    q2, k2, v2 = oracle.rope_qkv_f64(qkv, Hq, Hkv, positions=pt, lib=lib)
    assert np.array_equal(q1, q2) and np.array_equal(k1, k2) and np.array_equal(v1, v2)
    # each (i, i + d/2) pair keeps its length
    xin = heads[:, :, :Hq].transpose(0, 2, 1, 3)
    half = d // 2
    assert np.allclose(q1[..., :half] ** 2 + q1[..., half:] ** 2,
                       xin[..., :half] ** 2 + xin[..., half:] ** 2, rtol=1e-13)
    # q.k depends on the positions only through their difference
    base_pos = np.array([[3, 11, 40, 41, 100, 7]] * B, np.int32)
    qa, ka, _ = oracle.rope_qkv_f64(qkv, Hq, Hkv, positions=base_pos, lib=lib)
    qb, kb, _ = oracle.rope_qkv_f64(qkv, Hq, Hkv, positions=base_pos + 1234, lib=lib)
    dots_a = np.einsum("bhtd,bsd->bhts", qa, ka[:, 0])
    dots_b = np.einsum("bhtd,bsd->bhts", qb, kb[:, 0])
    assert np.allclose(dots_a, dots_b, rtol=1e-9, atol=1e-9)
    # d = 2: theta_0 = 1, a plain rotation by p radians
    x = np.array([[[0.3, -1.2, 0.5, 0.25, 2.0, -0.75]]])  # B=1, T=1, Hq=1, Hkv=1, d=2
    p = 3
    q, k, v = oracle.rope_qkv_f64(x, 1, 1, positions=np.array([[p]], np.int32), lib=lib)
    c, s_ = math.cos(p), math.sin(p)
    assert np.allclose(q[0, 0, 0], [0.3 * c + 1.2 * s_, 0.3 * s_ - 1.2 * c], rtol=0, atol=1e-15)
    assert np.allclose(k[0, 0, 0], [0.5 * c - 0.25 * s_, 0.5 * s_ + 0.25 * c], rtol=0, atol=1e-15)
    assert np.array_equal(v[0, 0, 0], [2.0, -0.75])


# ---------------------------------------------------------------- varlen
def pin_varlen_library(lib):
    """Packed sequences against torch SDPA (float64) over the whole packed
    batch with a block-diagonal (and causal) mask: no sequence sees another."""
    for seed, (lens, Hq, Hkv, d, causal) in enumerate([([5, 1, 9, 0, 3], 4, 2, 8, True),
                                                        ([7, 7, 2], 2, 2, 16, False),
                                                        ([12, 4], 6, 2, 8, True)]):
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        total = int(cu[-1])
        q = _rand((total, Hq, d), 1100 + seed)
        k = _rand((total, Hkv, d), 1110 + seed)
        v = _rand((total, Hkv, d), 1120 + seed)
        scale = 0.37
        o, lse = oracle.attn_fwd_varlen_f64(q, k, v, cu, causal=causal, scale=scale, lib=lib)
        seq = np.repeat(np.arange(len(lens)), lens)
        allowed = seq[:, None] == seq[None, :]
        if causal:
            allowed &= np.arange(total)[None, :] <= np.arange(total)[:, None]
        G = Hq // Hkv
        qt = torch.from_numpy(q).permute(1, 0, 2)
        kt = torch.from_numpy(k).repeat_interleave(G, dim=1).permute(1, 0, 2)
        vt = torch.from_numpy(v).repeat_interleave(G, dim=1).permute(1, 0, 2)
        want = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(allowed), scale=scale).permute(1, 0, 2)
        assert np.allclose(o, want.numpy(), rtol=0, atol=1e-12), seed
        logits = scale * torch.einsum("htd,hsd->hts", qt, kt)
        logits = logits.masked_fill(~torch.from_numpy(allowed), -math.inf)
        assert np.allclose(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_varlen_equal_lengths(lib):
    """Equal lengths: the packed result is the fixed-length batch's, exactly."""
    B, T, Hq, Hkv, d = 3, 6, 4, 2, 8
    q = _rand((B, Hq, T, d), 1130)
    k = _rand((B, Hkv, T, d), 1131)
    v = _rand((B, Hkv, T, d), 1132)
    o, lse = oracle.attn_fwd_f64(q, k, v, causal=True, scale=0.5, lib=lib)
    pack = lambda x: x.transpose(0, 2, 1, 3).reshape(B * T, x.shape[1], d)
    cu = np.arange(B + 1, dtype=np.int32) * T
    ov, lv = oracle.attn_fwd_varlen_f64(pack(q), pack(k), pack(v), cu, causal=True, scale=0.5,
                                        lib=lib)
    assert np.array_equal(ov, pack(o))
    assert np.array_equal(lv, lse.transpose(1, 0, 2).reshape(Hq, B * T))


def pin_threaded_forward(lib):
    """The all-core driver gives, bit for bit, the full fp64 entry's result,
    whatever the thread count and run length (a ragged run length, rows of
    several heads and batches, causal and full)."""
    from causal_gqa_attention_03_b200.inputs import make_qkv, bf16_bits
    B, Hq, Hkv, T, d = 2, 6, 2, 203, 32
    q, k, v = make_qkv(B, Hq, Hkv, T, d, seed=17, sigma_qk=2.5)
    scale = 0.2
    for causal in (True, False):
        o, lse = oracle.attn_fwd_f64(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                     causal=causal, scale=scale, lib=lib)
        for threads, run_rows in ((1, 256), (3, 37), (8, 64)):
            to, tl = oracle.attn_fwd_bf16_threaded(bf16_bits(q), bf16_bits(k), bf16_bits(v),
                                                   causal=causal, scale=scale, threads=threads,
                                                   run_rows=run_rows, lib=lib)
            assert np.array_equal(to, o) and np.array_equal(tl, lse)
    # the runs cover every row exactly once, and their flop counts sum to the
    # closed form 4 d sum_i (i + 1) = 2 d T (T + 1) per head
    runs = oracle.fwd_runs(B, Hq, T, True, 37)
    seen = np.zeros((B, Hq, T), dtype=int)
    for b, h, i0, i1 in runs:
        seen[b, h, i0:i1] += 1
    assert np.all(seen == 1)
    total = sum(oracle.run_flops(r, d, T, True) for r in runs)
    assert total == B * Hq * 2.0 * d * T * (T + 1)
    assert sum(oracle.run_flops(r, d, T, False) for r in runs) == B * Hq * 4.0 * d * T * T


def pin_threaded_backward(lib):
    """The per-slice threaded backward gives, bit for bit, one call's result."""
    B, Hq, Hkv, T, d = 2, 6, 2, 37, 16
    q = _rand((B, Hq, T, d), 1201, 1.5)
    k = _rand((B, Hkv, T, d), 1202, 1.5)
    v = _rand((B, Hkv, T, d), 1203)
    g = _rand((B, Hq, T, d), 1204)
    for causal in (True, False):
        ref = oracle.attn_bwd_f64(q, k, v, g, causal=causal, scale=0.3, lib=lib)
        for threads in (1, 4):
            got = oracle.attn_bwd_threaded(q, k, v, g, causal=causal, scale=0.3,
                                           threads=threads, lib=lib)
            for r, x in zip(ref, got):
                assert np.array_equal(r, x)


ALL_PINS = [pin_varlen_library, pin_varlen_equal_lengths, pin_rmsnorm_library, pin_rmsnorm_invariants, pin_rope_complex,
            pin_rope_invariants, pin_closed_forms, pin_library_sdpa, pin_decimal_large_logits, pin_invariants,
            pin_rows_entry, pin_bwd_library_autograd, pin_bwd_finite_differences,
            pin_bwd_invariants, pin_bwd_dq_rows_entry, pin_decode_library,
            pin_decode_invariants, pin_threaded_forward, pin_threaded_backward]
