"""tessera_attn_bwd_noalloc: the backward with the library's own static scratch
array instead of a caller workspace.

The file is collected last so that it runs after every other test as well as
alone; its GPU tests compare the entry point with tessera_attn_bwd on two
calls in a row (different problems, the second reusing the scratch the first
wrote) and on the largest synthetic workload.
"""
import math

import pytest
import torch

import causal_gqa_attention_03_b200 as tess
from causal_gqa_attention_03_b200 import inputs

ALIGNED = 0x10000000
TOO_LARGE = 6


def test_noalloc_too_large_is_rejected_before_any_cuda_call():
    lib = tess.load_library()
    assert lib is not None
    cap = tess.tessera_attn_bwd_noalloc_max_workspace_bytes()
    assert cap == 16 << 20
    B, Hq, Hkv, T, d = 1, 64, 8, 131072, 128
    assert tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d) > cap
    ptrs = [ALIGNED + i * (1 << 34) for i in range(9)]
    st = tess.tessera_attn_bwd_noalloc(*ptrs, B, Hq, Hkv, T, d, 1, 0.1, None)
    assert st == TOO_LARGE
    assert tess.tessera_status_str(st) != "unknown status"
    assert tess.tessera_attn_last_launch_count() == 0


def _both(q, k, v, g, causal, scale):
    o, lse = tess.attn_fwd(q, k, v, causal=causal, scale=scale)
    ref = [t.clone() for t in tess.attn_bwd(q, k, v, o, lse, g, causal=causal, scale=scale)]
    got = tess.attn_bwd_noalloc(q, k, v, o, lse, g, causal=causal, scale=scale)
    torch.cuda.synchronize()
    # the balanced dK/dV form (a fourth launch) applies when its workspace,
    # asked for by tessera_attn_bwd_workspace_bytes_kv, fits in the array
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    kv = tess.tessera_attn_bwd_workspace_bytes_kv(B, Hq, Hkv, T, d)
    balanced = (kv > tess.tessera_attn_bwd_workspace_bytes(B, Hq, T, d)
                and kv <= tess.tessera_attn_bwd_noalloc_max_workspace_bytes())
    assert tess.tessera_attn_last_launch_count() == (4 if balanced else 3)
    assert tess.tessera_attn_device_error() == 0
    return ref, got


def _same(ref, got, what):
    # Both entry points run the same three launches on the same data, and no
    # gradient is summed with atomics: dQ, dK and dV must agree bit for bit.
    # A stale row of the scratch array would show up here.
    for r, g_, name in zip(ref, got, ("dQ", "dK", "dV")):
        assert torch.equal(r, g_), f"{what}: {name} differs"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    cases = [(1, 8, 2, 1000, 128, True), (2, 4, 4, 513, 64, True), (1, 6, 3, 300, 128, False)]
    for n, (B, Hq, Hkv, T, d, causal) in enumerate(cases):
        q, k, v = (t.to(dev) for t in inputs.make_qkv(B, Hq, Hkv, T, d, seed=60 + n,
                                                      sigma_qk=1.5))
        g = inputs.make_grad(B, Hq, T, d, seed=70 + n).to(dev)
        ref, got = _both(q, k, v, g, causal, 1.0 / math.sqrt(d))
        _same(ref, got, (B, Hq, Hkv, T, d, causal))


@pytest.mark.gpu
def test_noalloc_largest_workload():
    dev = torch.device("cuda:0")
    w = inputs.WORKLOADS[inputs.LARGEST]
    assert (tess.tessera_attn_bwd_workspace_bytes(w.B, w.Hq, w.T, w.d)
            <= tess.tessera_attn_bwd_noalloc_max_workspace_bytes())
    q, k, v = (t.to(dev) for t in inputs.workload_inputs(w))
    g = inputs.workload_grad(w).to(dev)
    ref, got = _both(q, k, v, g, True, w.scale)
    _same(ref, got, w.name)
