"""Rotary position embedding with Position Interpolation (s2attn_rope_pi), the step just before
the attention (LongLoRA summary page, §3 "Phase 1" step 2 and §4 "Model setup"): the CUDA
kernel against the oracle's rope_pi element by element, in place and on packed-qkv views, and
composed with the S²-Attn forward and backward (gradients rotated back with the inverse)."""
import numpy as np
import pytest
import torch

from oracle import s2attn_oracle as orc
import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import make_inputs, to_f64

from gpu_helpers import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.lib()


def _x(B, N, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, N, H, d, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("B,N,H,d,base,pi", [
    (1, 256, 4, 64, 10000.0, 1.0),       # plain RoPE
    (2, 320, 8, 128, 10000.0, 0.5),      # 4k -> 8k interpolation, ragged N, batch 2
    (1, 8192, 8, 128, 10000.0, 0.5),     # the metric workload's sequence
    (1, 100000, 2, 128, 10000.0, 0.04),  # 100k context of the 7B model (4096 / 102400)
])
@pytest.mark.parametrize("inverse", [False, True])
def test_rope_matches_oracle(B, N, H, d, base, pi, inverse):
    x = _x(B, N, H, d, 7 + N)
    y = s2.rope_pi(x.cuda(), base=base, pi_scale=pi, inverse=inverse).cpu()
    ref = orc.rope_pi(to_f64(x), base=base, pi_scale=pi, inverse=inverse)
    assert_close("rope", y, ref)


def test_rope_in_place_and_on_packed_qkv():
    """In place, and on q and k inside a packed [B, N, 3, H, d] buffer, the result is
    bit-identical to the out-of-place call on contiguous copies; v is untouched."""
    B, N, H, d = 2, 256, 4, 128
    qkv = _x(B, N, 3 * H, d, 3).reshape(B, N, 3, H, d).cuda()
    want_q = s2.rope_pi(qkv[:, :, 0].contiguous(), pi_scale=0.5)
    want_k = s2.rope_pi(qkv[:, :, 1].contiguous(), pi_scale=0.5)
    v_before = qkv[:, :, 2].clone()
    for j in (0, 1):
        view = qkv[:, :, j]
        s2.s2attn_rope_pi(view, view, pi_scale=0.5)
    torch.cuda.synchronize()
    assert torch.equal(qkv[:, :, 0], want_q)
    assert torch.equal(qkv[:, :, 1], want_k)
    assert torch.equal(qkv[:, :, 2], v_before)
    x = _x(1, 64, 2, 64, 5).cuda()
    y = s2.rope_pi(x, pi_scale=0.25)
    s2.s2attn_rope_pi(x, x, pi_scale=0.25)
    assert torch.equal(x, y)


def test_rope_then_s2attn_forward_and_backward():
    """The attention layer with its position embedding: q, k rotated (PI 4k -> 8k), S²-Attn
    forward and backward, dq and dk rotated back with the inverse. Against the oracle's
    composition: s2attn_forward / s2attn_backward, then rope_pi(inverse) (the chain rule of an
    orthogonal map). The rotation itself is checked against the oracle above; as with every
    other bf16 input, both sides attend over the same rotated bf16 values (the kernel's),
    since the LSE bound of 1e-4 leaves no room for re-rounding q and k."""
    B, Hq, Hkv, N, d, G = 1, 4, 2, 512, 128, 128
    pi = 0.5
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, 2024, 1.0)
    scale = d ** -0.5
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    qr, kr = s2.rope_pi(qd, pi_scale=pi), s2.rope_pi(kd, pi_scale=pi)
    o, lse = s2.fwd(qr, kr, vd, G, scale)
    dqr, dkr, dv = s2.bwd(qr, kr, vd, o, lse, dod, G, scale)
    dq = s2.rope_pi(dqr, pi_scale=pi, inverse=True)
    dk = s2.rope_pi(dkr, pi_scale=pi, inverse=True)
    torch.cuda.synchronize()
    vf, dof = to_f64(v), to_f64(do)
    qrf, krf = to_f64(qr.cpu()), to_f64(kr.cpu())
    o_ref, lse_ref = orc.s2attn_forward(qrf, krf, vf, G, scale)
    dq_r, dk_r, dv_ref = orc.s2attn_backward(qrf, krf, vf, dof, G, scale)
    dq_ref = orc.rope_pi(dq_r, pi_scale=pi, inverse=True)
    dk_ref = orc.rope_pi(dk_r, pi_scale=pi, inverse=True)
    for name, g, r in (("o", o, o_ref), ("lse", lse, lse_ref), ("dq", dq, dq_ref),
                       ("dk", dk, dk_ref), ("dv", dv, dv_ref)):
        assert_close(name, g.cpu(), r)


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d,shift,flags,pi", [
    (1, 8, 8, 2048, 512, 128, None, 0, 0.5),     # Llama-like heads, PI 4k -> 8k
    (2, 4, 2, 640, 128, 64, None, 0, 1.0),       # d = 64 (two rows per lane step), GQA, batch 2
    (1, 4, 2, 512, 128, 128, 37, 2, 0.25),       # a roll of 37 under Variant 3: tiles of 3 runs
    (1, 4, 4, 300, 75, 64, None, 0, 0.5),        # odd G, roll 37, ragged end (rows past N)
])
def test_fused_rope_q_forward(B, Hq, Hkv, N, G, d, shift, flags, pi):
    """s2attn_fwd_rope_q: the queries' RoPE-PI fused into the forward's query-tile path. The
    rotated queries it writes match the oracle's rope_pi as closely as the standalone kernel's
    do (run starts are computed as there, later rows by angle addition, which avoids the fp32
    rounding of large angles); O and LSE match the oracle's attention over those rotated values;
    rotating in place gives the same bits."""
    q, k, v, _ = make_inputs(B, Hq, Hkv, N, d, 77 + N, 1.0)
    scale = d ** -0.5
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    kr = s2.rope_pi(kd, pi_scale=pi)
    o, lse = torch.empty_like(qd), torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    qr = torch.empty_like(qd)
    s2.s2attn_fwd_rope_q(qd, kr, vd, o, lse, qr, G, scale, shift=shift, flags=flags, pi_scale=pi)
    torch.cuda.synchronize()
    st, code = s2.s2attn_get_device_error()
    assert st == s2.S2ATTN_OK, (st, code)
    # the rotated queries: as close to the exact rotation as the standalone kernel's
    q_ref = orc.rope_pi(to_f64(q), pi_scale=pi)
    fused_err = assert_close("q_rot", qr.cpu(), q_ref)["max_abs"]
    alone_err = assert_close("q_rot", s2.rope_pi(qd, pi_scale=pi).cpu(), q_ref)["max_abs"]
    assert fused_err <= alone_err * 1.25 + 1e-3, (fused_err, alone_err)
    wrap = bool(flags & s2.S2ATTN_FLAG_WRAP_OWN_GROUP)
    front = bool(flags & s2.S2ATTN_FLAG_WRAP_FRONT_FIRST)
    o_ref, lse_ref = orc.s2attn_forward(to_f64(qr.cpu()), to_f64(kr.cpu()), to_f64(v), G, scale,
                                        shift=shift, wrap_own_group=wrap, wrap_front_first=front)
    assert_close("o", o.cpu(), o_ref)
    assert_close("lse", lse.cpu(), lse_ref)
    # in place: q_rot = q
    o2, lse2 = torch.empty_like(o), torch.empty_like(lse)
    s2.s2attn_fwd_rope_q(qd, kr, vd, o2, lse2, qd, G, scale, shift=shift, flags=flags, pi_scale=pi)
    torch.cuda.synchronize()
    assert torch.equal(qd, qr) and torch.equal(o2, o) and torch.equal(lse2, lse)
