"""Parity of the CUDA paged-KV decode step with the fp64 oracle, through the C
ABI, on a B200.

Tolerance: the forward's (the step is the forward's attention for one query
row, with bf16 inputs and output): max |err| <= 2e-2 and mean |err| <= 2e-3 on
O (bf16), |err| <= 1e-3 on LSE (fp32).

* small batches (ragged lengths across the 128-token chunk boundaries, empty
  sequences, G = 1 .. 16, d = 64 / 128, block sizes 8 .. 256): every element;
* the measured serving workload: every output of sampled sequences, checked
  by the oracle on a compact copy of their blocks;
* placement invariance: the same tokens under another block permutation or
  another block size give the same bits;
* the causal forward's last row over the same keys and values;
* device-side checks of lengths and block ids (errors reported, nothing read
  outside the cache).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu

O_MAX, O_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    tess.load_library()
    assert tess.tessera_attn_device_error() == 0


def run_decode(q, kc, vc, table, lens, max_seq_len=None, scale=None):
    """Host inputs in (table/lens numpy int32); (o fp32, lse fp32) host out."""
    t = torch.from_numpy(np.ascontiguousarray(table, dtype=np.int32)).to(DEV)
    n = torch.from_numpy(np.ascontiguousarray(lens, dtype=np.int32)).to(DEV)
    o, lse = tess.attn_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), t, n, max_seq_len=max_seq_len,
                              scale=scale)
    torch.cuda.synchronize()
    return o.float().cpu(), lse.cpu()


def check(o, lse, ro, rlse, what):
    o = o.double().numpy()
    lse = lse.double().numpy()
    err = np.abs(o - ro)
    assert np.all(np.isfinite(o)), what
    assert err.max() <= O_MAX, f"{what}: O max err {err.max():.3e}"
    assert err.mean() <= O_MEAN, f"{what}: O mean err {err.mean():.3e}"
    fin = np.isfinite(rlse)
    assert np.array_equal(fin, np.isfinite(lse)), what
    assert np.all(lse[~fin] == -np.inf), what
    if fin.any():
        e = np.abs(lse[fin] - rlse[fin]).max()
        assert e <= LSE_MAX, f"{what}: LSE max err {e:.3e}"


# (B, Hq, Hkv, d, bs, lengths)
CASES = [
    (3, 4, 2, 128, 16, [1, 127, 128]),
    (4, 8, 2, 128, 16, [129, 255, 256, 1000]),
    (2, 8, 8, 64, 8, [300, 17]),           # G = 1
    (3, 6, 2, 128, 32, [0, 513, 64]),      # G = 3, an empty sequence
    (2, 8, 1, 64, 64, [777, 1]),           # G = 8
    (2, 16, 1, 128, 16, [400, 129]),       # G = 16: two CTAs per chunk
    (2, 4, 2, 128, 256, [700, 256]),       # blocks larger than a chunk
    (1, 12, 4, 64, 128, [1025]),           # G = 3, d = 64
    (5, 4, 4, 128, 8, [5, 0, 131, 2048, 64]),
    (2, 16, 2, 128, 64, [1000, 77]),       # G = 8: eight heads per item
    (1, 32, 1, 128, 16, [300]),            # G = 32: two items of 16 heads
    (2, 6, 2, 64, 16, [0, 0]),             # every sequence empty
]


@pytest.mark.parametrize("B,Hq,Hkv,d,bs,lens", CASES)
def test_decode_every_element(B, Hq, Hkv, d, bs, lens):
    q, kc, vc, table, sl = inputs.make_paged(B, Hq, Hkv, d, bs, lens, seed=500 + sum(lens) + d,
                                             sigma_qk=1.5)
    scale = 1.0 / math.sqrt(d)
    o, lse = run_decode(q, kc, vc, table, sl)
    ro, rlse = oracle.paged_decode_f64(q.double().numpy(), kc.double().numpy(),
                                       vc.double().numpy(), table, sl, scale=scale)
    check(o, lse, ro, rlse, (B, Hq, Hkv, d, bs, lens))
    for b, n in enumerate(sl):
        if n == 0:
            assert not o[b].any() and torch.all(lse[b] == -math.inf)


def test_decode_large_logits_and_long_sequence():
    # Q/K sigma 4 (the headline forward's large logits) over 16384 tokens
    q, kc, vc, table, sl = inputs.make_paged(2, 8, 2, 128, 16, [16384, 9000], seed=77,
                                             sigma_qk=4.0)
    o, lse = run_decode(q, kc, vc, table, sl)
    ro, rlse = oracle.paged_decode_f64(q.double().numpy(), kc.double().numpy(),
                                       vc.double().numpy(), table, sl)
    check(o, lse, ro, rlse, "sigma 4, 16384 tokens")


def test_decode_serving_workload_sampled_sequences():
    w = inputs.DECODE
    q, kc, vc, table_d, lens_d = inputs.make_paged_device(w, DEV)
    o, lse = tess.attn_decode(q, kc, vc, table_d, lens_d, max_seq_len=w.max_len, scale=w.scale)
    torch.cuda.synchronize()
    assert tess.tessera_attn_last_launch_count() == 2
    assert tess.tessera_attn_device_error() == 0
    table, lens = table_d.cpu().numpy(), lens_d.cpu().numpy()
    rng = np.random.default_rng(5)
    rows = sorted({int(np.argmax(lens)), int(np.argmin(lens))} |
                  {int(x) for x in rng.choice(w.B, 4, replace=False)})
    sk, sv, st, sn = inputs.gather_sequences(table, lens, rows, w.bs, kc, vc)
    ro, rlse = oracle.paged_decode_f64(q[rows].double().cpu().numpy(), sk.double().numpy(),
                                       sv.double().numpy(), st, sn, scale=w.scale)
    check(o[rows].float().cpu(), lse[rows].cpu(), ro, rlse, f"{w.name} rows {rows}")


def test_decode_placement_and_block_size_do_not_change_bits():
    B, Hq, Hkv, d = 3, 8, 2, 128
    lens = [1000, 129, 300]
    q, kc, vc, table, sl = inputs.make_paged(B, Hq, Hkv, d, 16, lens, seed=91)
    base = run_decode(q, kc, vc, table, sl)
    # another permutation of the same blocks
    nb = kc.shape[0]
    perm = torch.randperm(nb, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(nb)
    t2 = np.where(table >= 0, inv.numpy()[np.maximum(table, 0)], -1).astype(np.int32)
    kc2 = torch.empty_like(kc)
    vc2 = torch.empty_like(vc)
    kc2[inv] = kc
    vc2[inv] = vc
    got = run_decode(q, kc2, vc2, t2, sl)
    assert torch.equal(base[0], got[0]) and torch.equal(base[1], got[1])
    # the same tokens in blocks of 8 (each block of 16 split in two)
    kc8 = kc.reshape(nb, Hkv, 2, 8, d).permute(0, 2, 1, 3, 4).reshape(2 * nb, Hkv, 8, d)
    vc8 = vc.reshape(nb, Hkv, 2, 8, d).permute(0, 2, 1, 3, 4).reshape(2 * nb, Hkv, 8, d)
    t8 = np.full((B, 2 * table.shape[1]), -1, dtype=np.int32)
    t8[:, 0::2] = np.where(table >= 0, 2 * table, -1)
    t8[:, 1::2] = np.where(table >= 0, 2 * table + 1, -1)
    got8 = run_decode(q, kc8.contiguous(), vc8.contiguous(), t8, sl)
    assert torch.equal(base[0], got8[0]) and torch.equal(base[1], got8[1])


def test_decode_matches_causal_forward_last_row():
    # one query row over n cached tokens = the causal forward's row n-1 when
    # that row's q is the query and the cache holds the same keys and values
    B, Hq, Hkv, T, d = 2, 8, 2, 777, 128
    q4, k4, v4 = inputs.make_qkv(B, Hq, Hkv, T, d, seed=93)
    of, lf = tess.attn_fwd(q4.to(DEV), k4.to(DEV), v4.to(DEV), causal=True)
    bs = 16
    nblk = (T + bs - 1) // bs
    pad = nblk * bs - T
    kp = torch.nn.functional.pad(k4, (0, 0, 0, pad))
    vp = torch.nn.functional.pad(v4, (0, 0, 0, pad))
    kc = kp.reshape(B, Hkv, nblk, bs, d).permute(0, 2, 1, 3, 4).reshape(B * nblk, Hkv, bs, d)
    vc = vp.reshape(B, Hkv, nblk, bs, d).permute(0, 2, 1, 3, 4).reshape(B * nblk, Hkv, bs, d)
    table = np.arange(B * nblk, dtype=np.int32).reshape(B, nblk)
    o, lse = run_decode(q4[:, :, T - 1].contiguous(), kc.contiguous(), vc.contiguous(), table,
                        np.full(B, T, dtype=np.int32))
    torch.cuda.synchronize()
    assert torch.allclose(o, of[:, :, T - 1].float().cpu(), atol=2e-2)
    assert torch.allclose(lse, lf[:, :, T - 1].cpu(), atol=1e-3)


def test_decode_no_sequences_and_all_empty():
    q, kc, vc, table, sl = inputs.make_paged(2, 4, 2, 64, 8, [0, 0], seed=5)
    o, lse = run_decode(q, kc, vc, table, sl, max_seq_len=0)
    assert tess.tessera_attn_last_launch_count() == 1  # the merge only
    assert not o.any() and torch.all(lse == -math.inf)
    o, lse = run_decode(q, kc, vc, table, sl)
    assert tess.tessera_attn_last_launch_count() == 2
    assert not o.any() and torch.all(lse == -math.inf)
    # B = 0 launches nothing
    st = tess.tessera_attn_decode(q.data_ptr(), 16, 16, 16, 16, 16, None, None, 0, 0, 4, 2, 64,
                                  8, 1, 1, 0, 0.1, None)
    assert st == 0 and tess.tessera_attn_last_launch_count() == 0


def test_decode_bad_lengths_and_block_ids_are_reported():
    B, Hq, Hkv, d, bs = 3, 4, 2, 128, 16
    lens = [300, 200, 100]
    q, kc, vc, table, sl = inputs.make_paged(B, Hq, Hkv, d, bs, lens, seed=95)
    ref_o, ref_lse = run_decode(q, kc, vc, table, sl)
    assert tess.tessera_attn_device_error() == 0
    # a length above max_seq_len: that sequence is empty, the others unchanged
    bad = sl.copy()
    bad[1] = 301
    o, lse = run_decode(q, kc, vc, table, bad, max_seq_len=300)
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_DECODE_INPUT
    assert not o[1].any() and torch.all(lse[1] == -math.inf)
    assert torch.equal(o[0], ref_o[0]) and torch.equal(o[2], ref_o[2])
    # a negative length
    bad = sl.copy()
    bad[2] = -5
    o, lse = run_decode(q, kc, vc, table, bad)
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_DECODE_INPUT
    assert not o[2].any() and torch.equal(o[0], ref_o[0])
    # a block id past the cache among sequence 0's tokens 144..159 (the chunk
    # holding it is dropped, the rest of the sequence still counts)
    t2 = table.copy()
    t2[0, 9] = kc.shape[0] + 1000
    o, lse = run_decode(q, kc, vc, t2, sl)
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_DECODE_INPUT
    assert torch.all(torch.isfinite(o[0])) and torch.equal(o[1], ref_o[1])
    # ... and negative ones for every block of sequence 2 (all of it is dropped)
    t2 = table.copy()
    t2[2, :(lens[2] + bs - 1) // bs] = -7
    o, lse = run_decode(q, kc, vc, t2, sl)
    assert tess.tessera_attn_device_error() == tess.DEVICE_ERR_DECODE_INPUT
    assert not o[2].any() and torch.equal(o[0], ref_o[0])
    # the error word is clear again
    run_decode(q, kc, vc, table, sl)
    assert tess.tessera_attn_device_error() == 0


def test_decode_writes_only_its_outputs():
    B, Hq, Hkv, d, bs = 2, 8, 2, 64, 16
    q, kc, vc, table, sl = inputs.make_paged(B, Hq, Hkv, d, bs, [200, 33], seed=97)
    pad = 4096
    ob = torch.full((B * Hq * d + 2 * pad,), 7.0, dtype=torch.bfloat16, device=DEV)
    lb = torch.full((B * Hq + 2 * pad,), 7.0, dtype=torch.float32, device=DEV)
    o = ob[pad:pad + B * Hq * d].view(B, Hq, d)
    lse = lb[pad:pad + B * Hq].view(B, Hq)
    tess.attn_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), torch.from_numpy(table).to(DEV),
                     torch.from_numpy(sl).to(DEV), out=o, lse=lse)
    torch.cuda.synchronize()
    assert tess.tessera_attn_device_error() == 0
    for b in (ob, lb):
        assert torch.all(b[:pad] == 7.0) and torch.all(b[-pad:] == 7.0)
    ro, rlse = oracle.paged_decode_f64(q.double().numpy(), kc.double().numpy(),
                                       vc.double().numpy(), table, sl)
    check(o.float().cpu(), lse.cpu(), ro, rlse, "guarded outputs")
