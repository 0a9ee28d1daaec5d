"""The C-ABI library on CPU: it loads, exports what the header declares, and
rejects bad arguments before touching the GPU (no compute calls here)."""
import glob
import os
import re

import pytest

import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import build as tbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    tbuild.build()
    return tess.load_library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_]\w*\s*\**\s*(tessera_\w+)\s*\(",
                            text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert "tessera_attn_fwd" in names
    assert set(names) == set(tess.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_has_no_fallback_to_the_oracle():
    # the product package never imports, loads or includes the oracle
    pkg = os.path.join(ROOT, "causal_gqa_attention_03_b200")
    bad = re.compile(r"^\s*(import|from)\s+oracle\b|liboracle|attn_ref|#include\s+\S*oracle",
                     re.M)
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h")):
            assert not bad.search(open(path).read()), path


ALIGNED = 0x10000000
GOOD = dict(q=ALIGNED, k=ALIGNED + 0x1000000, v=ALIGNED + 0x2000000, o=ALIGNED + 0x3000000,
            lse=ALIGNED + 0x4000000, B=1, Hq=4, Hkv=2, T=16, d=64, causal=1, scale=0.125,
            stream=None)


def call(**kw):
    a = dict(GOOD)
    a.update(kw)
    return tess.tessera_attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"],
                                 a["Hkv"], a["T"], a["d"], a["causal"], a["scale"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(T=-5), 1), (dict(Hq=0), 1), (dict(Hkv=0), 1),
    (dict(Hq=6, Hkv=4), 1), (dict(d=96), 2), (dict(d=256), 2), (dict(d=0), 2),
    (dict(scale=0.0), 1), (dict(scale=-0.5), 1), (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1), (dict(causal=2), 1),
    (dict(q=0), 1), (dict(k=0), 1), (dict(v=0), 1), (dict(o=0), 1),
    (dict(q=ALIGNED + 8), 3), (dict(o=ALIGNED + 0x3000002), 3), (dict(lse=ALIGNED + 0x4000004), 3),
    (dict(o=ALIGNED + 0x40), 1),           # O overlaps Q
    (dict(lse=ALIGNED + 0x3000000 + 64), 1),  # LSE overlaps O
    (dict(B=0), 0), (dict(T=0), 0),        # empty: nothing to launch
    (dict(B=0, q=0, k=0, v=0, o=0, lse=0), 0),
])
def test_argument_checks_before_any_cuda_call(lib, kw, status):
    assert call(**kw) == status
    if status != 0:
        assert tess.tessera_attn_last_launch_count() == 0


HOST = 0x7f0000000000  # host pointers are never dereferenced by a rejected call


def call_host(**kw):
    a = dict(GOOD, q_h=HOST, k_h=HOST + 0x1000000, v_h=HOST + 0x2000000, o_h=HOST + 0x3000000,
             lse_h=HOST + 0x4000000, chunks=0)
    a.update(kw)
    return tess.tessera_attn_fwd_host(a["q_h"], a["k_h"], a["v_h"], a["o_h"], a["lse_h"], a["q"],
                                      a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                                      a["T"], a["d"], a["causal"], a["scale"], a["chunks"],
                                      a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(Hq=6, Hkv=4), 1), (dict(d=96), 2), (dict(scale=0.0), 1),
    (dict(q=ALIGNED + 8), 3), (dict(o=ALIGNED + 0x40), 1),
    (dict(chunks=-1), 1), (dict(lse_h=0), 1), (dict(lse=0), 1),
    (dict(q_h=0), 1), (dict(k_h=0), 1), (dict(v_h=0), 1), (dict(o_h=0), 1),
    (dict(B=0), 0), (dict(T=0, q_h=0, o_h=0), 0),
])
def test_host_entry_argument_checks_before_any_cuda_call(lib, kw, status):
    assert call_host(**kw) == status
    assert tess.tessera_attn_last_launch_count() == 0


def plan_by_header_rule(B, Hq, Hkv, chunks):
    """The pieces of tessera_attn_fwd_host as its header states the rule."""
    slices, G = B * Hkv, Hq // Hkv
    target = chunks if chunks > 0 else 8
    if target <= slices:
        cuts = [slices * c // target for c in range(target + 1)]
        out = [(a, b, 0, G) for a, b in zip(cuts, cuts[1:]) if b > a]
    else:
        want = -(-target // slices)
        split = next((s for s in range(want, G) if G % s == 0), G)
        r = G // split
        out = [(sl, sl + 1, i * r, (i + 1) * r) for sl in range(slices) for i in range(split)]
    if chunks > 0:
        return out
    s0, s1, h0, h1 = out.pop()
    if s1 - s0 > 1:
        out.append((s0, s1 - 1, 0, G))
    tail = min(h1 - h0, 4)
    if h1 - tail > h0:
        out.append((s1 - 1, s1, h0, h1 - tail))
    return out + [(s1 - 1, s1, h, h + 1) for h in range(h1 - tail, h1)]


@pytest.mark.parametrize("B,Hq,Hkv", [(1, 32, 8), (1, 32, 1), (1, 32, 32), (4, 4, 4), (1, 2, 1),
                                      (3, 12, 4), (2, 6, 3), (64, 8, 8)])
@pytest.mark.parametrize("chunks", [0, 1, 3, 8, 40, 1000])
def test_host_plan_follows_the_rule_and_covers_every_head_once(lib, B, Hq, Hkv, chunks):
    plan = tess.tessera_attn_fwd_host_plan(B, Hq, Hkv, chunks)
    assert plan == plan_by_header_rule(B, Hq, Hkv, chunks)
    G = Hq // Hkv
    heads = []
    for s0, s1, h0, h1 in plan:
        assert (h0, h1) == (0, G) or (s1 == s0 + 1 and 0 <= h0 < h1 <= G)
        heads += [sl * G + h for sl in range(s0, s1) for h in range(h0, h1)]
    assert heads == list(range(B * Hq))


def test_host_plan_headline_shape_tapers_to_single_heads(lib):
    # [1, 32 | 8, T, d]: seven one-slice pieces, then the last slice head by head
    plan = tess.tessera_attn_fwd_host_plan(1, 32, 8, 0)
    assert plan == [(s, s + 1, 0, 4) for s in range(7)] + [(7, 8, h, h + 1) for h in range(4)]


@pytest.mark.parametrize("args", [(0, 8, 8, 0), (1, 8, 3, 0), (1, 8, 8, -1), (1, 0, 1, 0)])
def test_host_plan_rejects_bad_sizes(lib, args):
    n = lib.tessera_attn_fwd_host_plan(*args, None, 0)
    assert n == -1


def call_bwd(**kw):
    a = dict(GOOD, dout=ALIGNED + 0x5000000, dq=ALIGNED + 0x6000000, dk=ALIGNED + 0x7000000,
             dv=ALIGNED + 0x8000000, ws=ALIGNED + 0x9000000, ws_bytes=None)
    a.update(kw)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = tess.tessera_attn_bwd_workspace_bytes(a["B"], a["Hq"], a["T"], a["d"])
    return tess.tessera_attn_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"],
                                 a["dk"], a["dv"], a["ws"], a["ws_bytes"], a["B"], a["Hq"],
                                 a["Hkv"], a["T"], a["d"], a["causal"], a["scale"], a["stream"])


def test_bwd_workspace_bytes(lib):
    # D = rowsum(dO * O) in fp32, one value per query row
    assert tess.tessera_attn_bwd_workspace_bytes(2, 8, 100, 64) == 2 * 8 * 100 * 4
    assert tess.tessera_attn_bwd_workspace_bytes(1, 1, 1, 128) == 4
    assert tess.tessera_attn_bwd_workspace_bytes(1, 1, 1, 96) == 0
    # the balanced dK/dV form: D (256-byte aligned) + split * B*Hkv*T*d*2 fp32
    # when B*Hkv*ceil(T/128) < 512; split doubles while G allows, up to 8
    assert tess.tessera_attn_bwd_workspace_bytes_kv(1, 8, 1, 1000, 128) == \
        32000 + 8 * 1 * 1 * 1000 * 128 * 2 * 4
    assert tess.tessera_attn_bwd_workspace_bytes_kv(2, 6, 3, 300, 64) == \
        ((2 * 6 * 300 * 4 + 255) // 256) * 256 + 2 * 2 * 3 * 300 * 64 * 2 * 4
    for shape in [(1, 32, 8, 16384, 128), (2, 8, 8, 100, 64), (8, 32, 32, 2048, 128)]:
        B, Hq, Hkv, T, d = shape  # enough units, or G = 1: the three-kernel form
        assert tess.tessera_attn_bwd_workspace_bytes_kv(*shape) == \
            tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d)
    assert tess.tessera_attn_bwd_workspace_bytes_kv(1, 3, 2, 10, 64) == 0
    assert tess.tessera_attn_bwd_workspace_bytes_kv(1, 2, 1, 10, 96) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(Hq=6, Hkv=4), 1), (dict(d=96), 2), (dict(scale=0.0), 1),
    (dict(lse=0), 1), (dict(dout=0), 1), (dict(dq=0), 1), (dict(dk=0), 1), (dict(dv=0), 1),
    (dict(ws=0), 1), (dict(ws_bytes=16), 1),
    (dict(dout=ALIGNED + 0x5000008), 3), (dict(ws=ALIGNED + 0x9000004), 3),
    (dict(dq=ALIGNED + 0x40), 1),            # dQ overlaps Q
    (dict(dk=ALIGNED + 0x6000000), 1),       # dK overlaps dQ
    (dict(ws=ALIGNED + 0x5000000), 1),       # workspace overlaps dO
    (dict(B=0), 0), (dict(T=0), 0),
])
def test_bwd_argument_checks_before_any_cuda_call(lib, kw, status):
    assert call_bwd(**kw) == status
    if status != 0:
        assert tess.tessera_attn_last_launch_count() == 0


DEC = dict(q=ALIGNED, kc=ALIGNED + 0x1000000, vc=ALIGNED + 0x2000000, table=ALIGNED + 0x3000000,
           lens=ALIGNED + 0x3100000, o=ALIGNED + 0x4000000, lse=ALIGNED + 0x4100000,
           ws=ALIGNED + 0x5000000, ws_bytes=None, B=4, Hq=8, Hkv=2, d=128, bs=16, max_blocks=8,
           num_blocks=40, max_seq_len=128, scale=0.125, stream=None)


def call_decode(**kw):
    a = dict(DEC)
    a.update(kw)
    if a["ws_bytes"] is None:
        a["ws_bytes"] = tess.tessera_attn_decode_workspace_bytes(a["B"], a["Hq"],
                                                                 a["max_seq_len"], a["d"])
    return tess.tessera_attn_decode(a["q"], a["kc"], a["vc"], a["table"], a["lens"], a["o"],
                                    a["lse"], a["ws"], a["ws_bytes"], a["B"], a["Hq"], a["Hkv"],
                                    a["d"], a["bs"], a["max_blocks"], a["num_blocks"],
                                    a["max_seq_len"], a["scale"], a["stream"])


def test_decode_workspace_bytes(lib):
    # partial outputs and (max, sum) pairs per (sequence, head, 128-token slot),
    # then an int per item (at most one per head), rounded up to 16 bytes
    assert tess.tessera_attn_decode_workspace_bytes(4, 8, 128, 128) == 4 * 8 * 1 * 130 * 4 + 128
    assert tess.tessera_attn_decode_workspace_bytes(2, 4, 129, 64) == 2 * 4 * 2 * 66 * 4 + 32
    assert tess.tessera_attn_decode_workspace_bytes(1, 3, 1, 64) == 3 * 66 * 4 + 16
    assert tess.tessera_attn_decode_workspace_bytes(3, 4, 0, 64) == 0
    assert tess.tessera_attn_decode_workspace_bytes(1, 1, 1, 96) == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(Hq=6, Hkv=4), 1), (dict(Hkv=0), 1), (dict(d=96), 2),
    (dict(bs=12), 2), (dict(bs=4), 2), (dict(bs=0), 2), (dict(scale=float("nan")), 1),
    (dict(max_blocks=0), 1), (dict(num_blocks=0), 1), (dict(max_seq_len=-1), 1),
    (dict(max_seq_len=8 * 16 + 1), 1),                 # beyond the table's capacity
    (dict(num_blocks=1 << 26), 1),                     # rows past 32-bit TMA coordinates
    (dict(q=0), 1), (dict(kc=0), 1), (dict(table=0), 1), (dict(lens=0), 1), (dict(o=0), 1),
    (dict(ws=0), 1), (dict(ws_bytes=16), 1),
    (dict(q=ALIGNED + 8), 3), (dict(vc=ALIGNED + 0x2000004), 3),
    (dict(table=ALIGNED + 0x3000002), 3), (dict(ws=ALIGNED + 0x5000008), 3),
    (dict(o=ALIGNED + 0x40), 1),                       # o overlaps q
    (dict(lse=ALIGNED + 0x3000000), 1),                # lse overlaps the block table
    (dict(ws=ALIGNED + 0x4000000), 1),                 # workspace overlaps o
    (dict(B=0), 0),
])
def test_decode_argument_checks_before_any_cuda_call(lib, kw, status):
    assert call_decode(**kw) == status
    assert tess.tessera_attn_last_launch_count() == 0


@pytest.mark.parametrize("kw,status", [
    (dict(rows=-1), 1), (dict(dim=0), 1), (dict(eps=-1.0), 1), (dict(eps=float("inf")), 1),
    (dict(dim=12), 2), (dict(dim=8200), 2), (dict(dim=16384), 2),
    (dict(x=0), 1), (dict(w=0), 1), (dict(y=0), 1),
    (dict(x=ALIGNED + 8), 3), (dict(y=ALIGNED + 0x1000004), 3),
    (dict(y=ALIGNED + 0x40), 1),                     # y overlaps x (not in place)
    (dict(w=ALIGNED + 0x1000000 + 64), 1),           # w inside y
    (dict(rows=0), 0),
])
def test_rmsnorm_argument_checks_before_any_cuda_call(lib, kw, status):
    a = dict(x=ALIGNED, w=ALIGNED + 0x2000000, y=ALIGNED + 0x1000000, rows=16, dim=4096,
             eps=1e-6)
    a.update(kw)
    assert tess.tessera_rmsnorm(a["x"], a["w"], a["y"], a["rows"], a["dim"], a["eps"],
                                None) == status
    assert tess.tessera_attn_last_launch_count() == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(T=-1), 1), (dict(Hq=6, Hkv=4), 1), (dict(Hkv=0), 1),
    (dict(d=96), 2), (dict(d=32), 2), (dict(base=0.0), 1), (dict(base=float("nan")), 1),
    (dict(qkv=0), 1), (dict(q=0), 1), (dict(k=0), 1), (dict(v=0), 1),
    (dict(qkv=ALIGNED + 4), 3), (dict(k=ALIGNED + 0x2000008), 3), (dict(pos=ALIGNED + 0x5000002), 3),
    (dict(q=ALIGNED + 0x100), 1),                    # q overlaps qkv
    (dict(v=ALIGNED + 0x1000000), 1),                # v overlaps q
    (dict(pos=ALIGNED + 0x2000000), 1),              # positions inside k
    (dict(B=0), 0), (dict(T=0), 0),
])
def test_rope_argument_checks_before_any_cuda_call(lib, kw, status):
    a = dict(qkv=ALIGNED, pos=ALIGNED + 0x5000000, q=ALIGNED + 0x1000000, k=ALIGNED + 0x2000000,
             v=ALIGNED + 0x3000000, B=2, T=100, Hq=8, Hkv=2, d=128, base=10000.0)
    a.update(kw)
    assert tess.tessera_rope_qkv(a["qkv"], a["pos"], a["q"], a["k"], a["v"], a["B"], a["T"],
                                 a["Hq"], a["Hkv"], a["d"], a["base"], None) == status
    assert tess.tessera_attn_last_launch_count() == 0


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), 1), (dict(total=-1), 1), (dict(max_seqlen=-1), 1), (dict(Hq=6, Hkv=4), 1),
    (dict(d=96), 2), (dict(scale=0.0), 1), (dict(causal=2), 1),
    (dict(max_seqlen=5000), 1),                      # longer than total
    (dict(q=0), 1), (dict(o=0), 1), (dict(cu=0), 1),
    (dict(q=ALIGNED + 8), 3), (dict(lse=ALIGNED + 0x4000004), 3), (dict(cu=ALIGNED + 0x5000002), 3),
    (dict(o=ALIGNED + 0x100), 1),                    # o overlaps q
    (dict(lse=ALIGNED + 0x5000000), 1),              # lse overlaps cu_seqlens
    (dict(o=ALIGNED + 0x4000000), 1),                # o overlaps lse
    (dict(B=0), 0), (dict(total=0, max_seqlen=0), 0), (dict(max_seqlen=0), 0),
])
def test_varlen_argument_checks_before_any_cuda_call(lib, kw, status):
    a = dict(q=ALIGNED, k=ALIGNED + 0x1000000, v=ALIGNED + 0x2000000, o=ALIGNED + 0x3000000,
             lse=ALIGNED + 0x4000000, cu=ALIGNED + 0x5000000, B=3, total=4000, max_seqlen=2000,
             Hq=8, Hkv=2, d=128, causal=1, scale=0.1)
    a.update(kw)
    assert tess.tessera_attn_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"],
                                        a["B"], a["total"], a["max_seqlen"], a["Hq"], a["Hkv"],
                                        a["d"], a["causal"], a["scale"], None) == status
    assert tess.tessera_attn_last_launch_count() == 0


@pytest.mark.parametrize("limit_us", [0, 10_000_001, 2**32 - 1])
def test_selftest_rejects_bad_limits_before_any_cuda_call(lib, limit_us):
    assert tess.tessera_attn_selftest_timeout(limit_us, None) == 1


def test_status_strings(lib):
    for s in range(6):
        assert tess.tessera_status_str(s)
    assert tess.tessera_status_str(99) == "unknown status"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(tess, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(tess, "_lib", None)
    with pytest.raises(ImportError):
        tess.load_library()
