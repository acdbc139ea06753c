"""CUDA path vs the fp64 oracle, element by element, on seeded inputs (small and edge cases).

Every call goes through the C ABI (libs2attn.so); nothing here computes attention in torch.
"""
import zlib

import numpy as np
import pytest
import torch

import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import WORKLOADS, make_inputs

from gpu_helpers import assert_close, check_case, gpu_run, log_case, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.lib()


def test_small_workload():
    w = WORKLOADS["small_h4_n256_g64_d64"]
    check_case(w.B, w.Hq, w.Hkv, w.N, w.G, w.d, w.seed)


@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shb,shift,q_gain", [
    # ragged tail: N is not a multiple of the 128-row tile; GQA; batch 2
    ("ragged_gqa", 2, 4, 2, 320, 64, 64, None, None, 1.0),
    # groups straddle tiles and the roll splits tiles (G/2 = 96)
    ("straddle", 1, 4, 4, 384, 192, 128, None, None, 1.0),
    # one group, no roll: full causal attention
    ("full_causal", 1, 2, 2, 256, 256, 128, 2, 0, 1.0),
    # MQA: one kv head read by rolled and unrolled query heads
    ("mqa_mixed", 1, 8, 1, 512, 128, 128, None, None, 1.0),
    # every head rolled, and rolled the other way ("shift up")
    ("pattern2_up", 1, 4, 2, 512, 256, 64, 0, 512 - 128, 1.0),
    # no head rolled ("short attention")
    ("pattern1", 1, 4, 4, 512, 128, 128, 4, 0, 1.0),
    # 8 groups per tile
    ("tiny_groups", 1, 2, 2, 256, 16, 64, None, None, 1.0),
    # a single short tile
    ("one_tile", 1, 2, 2, 16, 16, 128, None, None, 1.0),
    # several full tiles per group, rolled by a whole number of tiles
    ("aligned", 1, 2, 2, 2048, 512, 128, None, None, 1.0),
    # a group boundary inside a warp's 32 rows of a query tile whose first key tile lies
    # before that group: some rows of the warp see no key in their first step
    ("midwarp_groups", 1, 4, 2, 544, 136, 64, None, 64, 1.0),
])
def test_edge_cases(name, B, Hq, Hkv, N, G, d, shb, shift, q_gain):
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32(name.encode()) % 10000, shb=shb, shift=shift, q_gain=q_gain)


@pytest.mark.parametrize("mode", ["recompute", "per_kv_head", "phases"])
@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shb,shift", [
    ("ragged_gqa", 2, 4, 2, 320, 64, 64, None, None),       # unaligned slots, 2 kv heads
    ("straddle", 1, 4, 4, 384, 192, 128, None, None),       # roll splits tiles
    ("mqa_mixed", 1, 8, 1, 512, 128, 128, None, None),      # 8 query heads on one kv head
    ("aligned_gqa", 1, 8, 4, 2048, 512, 128, None, None),   # packed (triangular) slots
])
def test_backward_paths(mode, name, B, Hq, Hkv, N, G, d, shb, shift):
    """Each backward path — dQ recomputed, dS handed off one kv head per pass, and the dS
    stages called one at a time — against the oracle."""
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32((name + mode).encode()) % 10000, shb=shb,
               shift=shift, mode=mode)


def test_peaky_logits_forward():
    """Queries scaled by 4 make the logits peaky, so the running maximum of the online softmax
    grows by more than the rescale threshold inside rows: O and LSE at the stated bounds.

    The gradients of this input are four times the scale of the workloads' (dK = scale dS^T Q
    grows with the query gain) and are not held to the absolute bound stated for N(0, 1)
    inputs: rounding P and dS to bf16 and forming D from the bf16 O (what every flash-style
    bf16 backward does) already puts dK 0.098 and dQ 0.02 away from the exact values for this
    input. Their figures are logged with the others."""
    B, Hq, Hkv, N, G, d = 1, 4, 4, 1024, 256, 128
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, 3600, 4.0)
    scale = d ** -0.5
    g = gpu_run(q, k, v, do, G, scale)
    r = oracle_run(q, k, v, do, G, scale)
    report = {"o": assert_close("o", g["o"], r["o"]), "lse": assert_close("lse", g["lse"], r["lse"])}
    for name in ("dq", "dk", "dv"):
        dd = np.abs(g[name].double().numpy() - r[name])
        report[name] = {"max_abs": float(dd.max()), "mean_abs": float(dd.mean()),
                        "asserted": False}
    log_case({"test": "peaky_logits", "q_gain": 4.0}, report)


def test_shifted_head_equals_unshifted_on_rolled_input():
    """A rolled head equals an unrolled run on torch.roll-ed inputs, rolled back (bitwise)."""
    B, Hq, N, G, d = 1, 2, 1024, 256, 128
    q, k, v, do = make_inputs(B, Hq, Hq, N, d, 77)
    scale = d ** -0.5
    a = gpu_run(q, k, v, do, G, scale, shb=1, shift=G // 2)
    rq, rk, rv, rdo = (torch.roll(x, -G // 2, dims=1) for x in (q, k, v, do))
    b = gpu_run(rq, rk, rv, rdo, G, scale, shb=2, shift=0)
    for name in ("o", "dq", "dk", "dv"):
        back = torch.roll(b[name], G // 2, dims=1)
        assert torch.equal(a[name][:, :, 1], back[:, :, 1]), name
    assert torch.equal(a["lse"][:, 1], torch.roll(b["lse"], G // 2, dims=2)[:, 1])


def test_deterministic():
    w = WORKLOADS["small_h4_n256_g64_d64"]
    q, k, v, do = make_inputs(w.B, w.Hq, w.Hkv, 1024, 128, 5)
    a = gpu_run(q, k, v, do, 256, 0.1)
    b = gpu_run(q, k, v, do, 256, 0.1)
    for name in a:
        assert torch.equal(a[name], b[name]), name


def test_wait_timeout_is_reported_and_context_survives():
    s2.s2attn_selftest_wait_timeout(50_000_000)    # 50 ms
    st, code = s2.s2attn_get_device_error()
    assert st == s2.S2ATTN_ERR_TIMEOUT
    assert code == (4 << 8) | 1
    st, code = s2.s2attn_get_device_error()
    assert st == s2.S2ATTN_OK and code == 0
    check_case(1, 2, 2, 256, 64, 64, seed=3, backward=False)


def test_invalid_args_raise():
    q = torch.zeros(1, 256, 3, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(s2.S2AttnError):
        s2.fwd(q, q, q, 64)                         # odd head count with the default split
    q = torch.zeros(1, 256, 4, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(s2.S2AttnError):
        s2.fwd(q, q, q, 64)                         # unsupported head dim
