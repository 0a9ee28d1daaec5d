"""The fp64 oracle against its pins (CPU only).

Each pin checks the oracle against something other than itself (closed forms,
a library routine, exact Decimal arithmetic, invariants).  The planted-mistake
test then shows the pins have teeth: every plausible slip in the oracle's
source -- a dropped term, a wrong sign or index, a transposed operand --
makes at least one pin fail.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_empty_inputs(oracle_lib):
    for shape in [(0, 2, 5, 4), (1, 2, 0, 4)]:
        q = np.zeros(shape)
        kv = np.zeros((shape[0], 1, shape[2], shape[3]))
        o, lse = oracle.attn_fwd_f64(q, kv, kv, causal=True, scale=0.5, lib=oracle_lib)
        assert o.size == 0 and lse.size == 0


def test_invalid_arguments(oracle_lib):
    q = np.zeros((1, 3, 4, 2))
    kv = np.zeros((1, 2, 4, 2))  # Hq not a multiple of Hkv
    with pytest.raises(ValueError):
        oracle.attn_fwd_f64(q, kv, kv, lib=oracle_lib)
    rows = np.array([[0, 0, 4]])  # row index out of range
    qb = np.zeros((1, 2, 4, 2), np.uint16)
    kb = np.zeros((1, 1, 4, 2), np.uint16)
    with pytest.raises(ValueError):
        oracle.attn_rows_bf16(qb, kb, kb, rows, lib=oracle_lib)


# (description, text in attn_ref.c, replacement).  Each is a mistake a careful
# reader could plausibly make when writing the definition down.
MUTATIONS = [
    ("causal mask drops the diagonal", "causal ? (int64_t)i + 1 : (int64_t)T",
     "causal ? (int64_t)i : (int64_t)T"),
    ("causal mask one key too many", "causal ? (int64_t)i + 1 : (int64_t)T",
     "causal ? ((int64_t)i + 2 < T ? (int64_t)i + 2 : (int64_t)T) : (int64_t)T"),
    ("group mapping h % Hkv instead of h / G", "const int g = h / G;",
     "const int g = h % Hkv;"),
    ("no max subtraction", "s[j] = exp(s[j] - m);", "s[j] = exp(s[j]);"),
    ("max subtracted with the wrong sign", "s[j] = exp(s[j] - m);", "s[j] = exp(s[j] + m);"),
    ("LSE missing the max", "*lse = m + log(l);", "*lse = log(l);"),
    ("LSE in base 2", "*lse = m + log(l);", "*lse = m + log2(l);"),
    ("scale not applied", "s[j] = scale * dot;", "s[j] = dot;"),
    ("K used in place of V", "o[c] += s[j] * vh[j * d + c];", "o[c] += s[j] * kh[j * d + c];"),
    ("V indexed transposed", "o[c] += s[j] * vh[j * d + c];",
     "o[c] += s[j] * vh[(c % n_keys) * d + (j % d)];"),
    ("missing normalisation", "o[c] /= l;", "o[c] /= 1.0;"),
    ("query index off by one head row", "dot += q[c] * kh[j * d + c];",
     "dot += q[(c + 1) % d] * kh[j * d + c];"),
    ("bf16 widened with the wrong shift", "(uint32_t)bits << 16", "(uint32_t)bits << 15"),
    # backward
    ("backward drops D", "const double ds = p[j] * (dp - D);", "const double ds = p[j] * dp;"),
    ("backward adds D", "const double ds = p[j] * (dp - D);",
     "const double ds = p[j] * (dp + D);"),
    ("D from Q instead of O", "D += dout[c] * o[c];", "D += dout[c] * q[c];"),
    ("P not normalised by the LSE", "p[j] = exp(s[j] - lse);", "p[j] = exp(s[j]);"),
    ("dQ missing the scale", "dq[c] += scale * ds * kh[j * d + c];",
     "dq[c] += ds * kh[j * d + c];"),
    ("dK missing the scale", "dkh[j * d + c] += scale * ds * q[c];",
     "dkh[j * d + c] += ds * q[c];"),
    ("dK from dO instead of Q", "dkh[j * d + c] += scale * ds * q[c];",
     "dkh[j * d + c] += scale * ds * dout[c];"),
    ("dV weighted by dS instead of P", "dvh[j * d + c] += p[j] * dout[c];",
     "dvh[j * d + c] += ds * dout[c];"),
    ("backward ignores the causal mask", "const int64_t n_keys = causal ? i + 1 : T;",
     "const int64_t n_keys = T;"),
    ("backward group mapping h % Hkv", "((int64_t)b * Hkv + h / G)",
     "((int64_t)b * Hkv + h % Hkv)"),
    # paged decode
    ("decode row within the block from j / bs",
     "(((int64_t)blk * Hkv + g) * bs + j % bs) * d", "(((int64_t)blk * Hkv + g) * bs + (j / bs) % bs) * d"),
    ("decode cache heads reversed", "(((int64_t)blk * Hkv + g) * bs + j % bs) * d",
     "(((int64_t)blk * Hkv + (Hkv - 1 - g)) * bs + j % bs) * d"),
    ("decode gathers V from the K cache", "vh[j * d + c] = v_cache[src + c];",
     "vh[j * d + c] = k_cache[src + c];"),
    ("decode group mapping h % Hkv", "for (int h = g * G; h < (g + 1) * G; ++h) {",
     "for (int h = g; h < Hq; h += Hkv) {"),
    ("decode drops the last token", "attend_one_row(q + row * d, kh, vh, n, d, scale, s, o + row * d, &lse[row]);",
     "attend_one_row(q + row * d, kh, vh, n > 1 ? n - 1 : n, d, scale, s, o + row * d, &lse[row]);"),
    # prologue
    ("RMSNorm without eps", "1.0 / sqrt(ss / dim + eps)", "1.0 / sqrt(ss / dim)"),
    ("RMSNorm over the sum, not the mean", "1.0 / sqrt(ss / dim + eps)", "1.0 / sqrt(ss + eps)"),
    ("RMSNorm weight dropped", "yr[c] = xr[c] * inv * w[c];", "yr[c] = xr[c] * inv;"),
    ("RoPE rotates the other way", "y[i] = x[i] * c - x[i + half] * s;",
     "y[i] = x[i] * c + x[i + half] * s;"),
    ("RoPE pairs neighbours instead of halves", "y[i + half] = x[i] * s + x[i + half] * c;",
     "y[i + half] = x[i] * s + x[i + half] * c; if (i % 2 == 1) { double t_ = y[i]; y[i] = y[i - 1]; y[i - 1] = t_; }"),
    ("RoPE frequency exponent i / d", "pow(base, -2.0 * i / d)", "pow(base, -1.0 * i / d)"),
    ("RoPE positions off by one", ": (double)t;", ": (double)t + 1.0;"),
    ("RoPE leaves the keys unrotated",
     "rope_one_head(tok + (int64_t)(Hq + h) * d, p, d, base,", "rope_one_head(tok + (int64_t)(Hq + h) * d, 0.0, d, base,"),
    ("value heads taken from the key slot", "const double *src = tok + (int64_t)(Hq + Hkv + h) * d;",
     "const double *src = tok + (int64_t)(Hq + h) * d;"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(desc, old, new, tmp_path):
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {old!r}"
    mutant_src = tmp_path / "attn_ref_mutant.c"
    mutant_src.write_text(src.replace(old, new))
    mutant_lib = str(tmp_path / "libmutant.so")
    oracle.build(str(mutant_src), mutant_lib)
    lib = oracle.load(mutant_lib)
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            failures.append(pin.__name__)
    assert failures, f"no pin caught the planted mistake: {desc}"
