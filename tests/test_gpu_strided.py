"""Strided tensors (s2attn_fwd_general / s2attn_bwd_general): q, k, v as views of one packed
qkv buffer, the layout of LongLoRA's Algorithm 1, and gradients written into a packed dqkv,
also combined with the option flags (Table 8 variants, a partial last group).

The kernels only address differently, so the results must equal the contiguous path's bit for
bit; the small case is also checked against the oracle.
"""
import pytest
import torch

import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import make_inputs

from gpu_helpers import assert_close, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.lib()


def _run_contiguous(q, k, v, do, G, scale, flags=0):
    o, lse = s2.fwd(q, k, v, G, scale, flags=flags)
    dq, dk, dv = s2.bwd(q, k, v, o, lse, do, G, scale, flags=flags)
    return o, lse, dq, dk, dv


V2, V3 = s2.S2ATTN_FLAG_WRAP_OWN_GROUP, s2.S2ATTN_FLAG_WRAP_FRONT_FIRST
PARTIAL = s2.S2ATTN_FLAG_PARTIAL_LAST_GROUP


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d,flags", [
    (2, 4, 4, 320, 64, 64, 0), (1, 8, 2, 1024, 256, 128, 0), (1, 4, 4, 2048, 512, 128, 0),
    (2, 4, 2, 320, 64, 64, V2), (2, 4, 2, 320, 64, 64, V3), (1, 4, 4, 704, 256, 128, PARTIAL)])
def test_packed_qkv_matches_contiguous(B, Hq, Hkv, N, G, d, flags):
    dev = torch.device("cuda")
    q, k, v, do = (x.to(dev) for x in make_inputs(B, Hq, Hkv, N, d, 4242 + N))
    scale = d ** -0.5
    ref = _run_contiguous(q, k, v, do, G, scale, flags)
    # packed [B, N, Hq + 2 Hkv, d] buffers (token stride (Hq + 2 Hkv) d) for qkv and dqkv
    H3 = Hq + 2 * Hkv
    qkv = torch.empty(B, N, H3, d, dtype=torch.bfloat16, device=dev)
    qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:] = q, k, v
    qv, kv_, vv = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    assert not qv.is_contiguous()
    # O and dO interleaved with padding tokens: token stride 2 Hq d
    opad = torch.zeros(B, N, 2 * Hq, d, dtype=torch.bfloat16, device=dev)
    ov = opad[:, :, :Hq]
    dopad = torch.zeros(B, N, 2 * Hq, d, dtype=torch.bfloat16, device=dev)
    dopad[:, :, :Hq] = do
    dov = dopad[:, :, :Hq]
    lse = torch.empty(B, Hq, N, dtype=torch.float32, device=dev)
    s2.s2attn_fwd(qv, kv_, vv, ov, lse, G, scale, flags=flags)
    dqkv = torch.zeros(B, N, H3, d, dtype=torch.bfloat16, device=dev)
    dqv, dkv, dvv = dqkv[:, :, :Hq], dqkv[:, :, Hq:Hq + Hkv], dqkv[:, :, Hq + Hkv:]
    s2.s2attn_bwd(qv, kv_, vv, ov, lse, dov, dqv, dkv, dvv, G, scale, flags=flags)
    torch.cuda.synchronize()
    st, code = s2.s2attn_get_device_error()
    assert st == s2.S2ATTN_OK, hex(code)
    for name, a, b in (("o", ov, ref[0]), ("lse", lse, ref[1]), ("dq", dqv, ref[2]),
                       ("dk", dkv, ref[3]), ("dv", dvv, ref[4])):
        assert torch.equal(a, b), name
    # padding tokens of O were not touched
    assert torch.count_nonzero(opad[:, :, Hq:]) == 0
    if N <= 320:
        r = oracle_run(q.cpu(), k.cpu(), v.cpu(), do.cpu(), G, scale, flags=flags)
        assert_close("o", ov.cpu(), r["o"])
        assert_close("dq", dqv.cpu(), r["dq"])
        assert_close("dk", dkv.cpu(), r["dk"])
        assert_close("dv", dvv.cpu(), r["dv"])
