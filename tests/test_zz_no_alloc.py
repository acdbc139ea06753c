"""The allocation-free backward entry point, s2attn_bwd_noalloc.

Some callers cannot hand the library a workspace: a plugin host whose fixed call signature has
no scratch argument, or a latency-critical path that must not call cudaMalloc (it can
synchronise the device and fail under memory pressure). For them s2attn_bwd_noalloc keeps its
scratch in a static array inside the library. These tests call it through the C ABI and check
that it gives the same gradients as s2attn_bwd with a caller workspace and that both match the
fp64 oracle, on two calls in a row (the second on different inputs, so stale scratch contents
from the first cannot help); one shape fits all dS tiles in the array at once, the other needs
several dK/dV + dQ passes over it. A shape beyond the array's capacity is refused before any
launch.

The file name sorts last so that, in a run stopping at the first failure, every other test has
already run.
"""
import ctypes

import pytest
import torch

import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import make_inputs

from gpu_helpers import assert_close, oracle_run


def _c(t):
    return ctypes.c_void_p(t.data_ptr())


def _grads_with_workspace(lib, q, k, v, o, lse, do, G, scale):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(lib.s2attn_bwd_workspace_size(B, Hq, N), dtype=torch.uint8, device=q.device)
    st = lib.s2attn_bwd(_c(q), _c(k), _c(v), _c(o), _c(lse), _c(do), _c(dq), _c(dk), _c(dv),
                        B, Hq, Hkv, N, d, G, scale, _c(ws), ws.numel(),
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, s2.status_string(st)
    return dq, dk, dv


def _grads_no_alloc(lib, q, k, v, o, lse, do, G, scale):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib.s2attn_bwd_noalloc(_c(q), _c(k), _c(v), _c(o), _c(lse), _c(do), _c(dq), _c(dk),
                                _c(dv), B, Hq, Hkv, N, d, G, scale,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, s2.status_string(st)
    return dq, dk, dv


@pytest.mark.gpu
@pytest.mark.parametrize("B,Hq,Hkv,N,G,d", [
    (1, 8, 4, 2048, 512, 128),     # every kv head's dS tiles fit in the array: one pass
    (1, 32, 32, 4096, 1024, 128),  # 4.7 MB of dS tiles per kv head: several passes
])
def test_no_alloc_backward_matches_workspace_backward_and_oracle(B, Hq, Hkv, N, G, d):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = s2.lib()
    scale = d ** -0.5
    for seed in (11, 12):   # two calls in a row, different inputs
        qc, kc, vc, doc = make_inputs(B, Hq, Hkv, N, d, seed)
        q, k, v, do = (x.cuda() for x in (qc, kc, vc, doc))
        o, lse = s2.fwd(q, k, v, G, scale)
        ref = _grads_with_workspace(lib, q, k, v, o, lse, do, G, scale)
        got = _grads_no_alloc(lib, q, k, v, o, lse, do, G, scale)
        torch.cuda.synchronize()
        st, code = s2.s2attn_get_device_error()
        assert st == s2.S2ATTN_OK, (st, code)
        exact = oracle_run(qc, kc, vc, doc, G, scale, backward=True)
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            assert_close(name, a.cpu(), b.double().cpu().numpy())
            assert_close(name, a.cpu(), exact[name])


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    lib = s2.lib()
    A = 0x10000   # never dereferenced: the size check comes first
    # B*Hq*N = 4 * 32 * 32768 = 4,194,304 rows > 2,097,152
    st = lib.s2attn_bwd_noalloc(*([A] * 9), 4, 32, 32, 32768, 128, 8192, 0.088, None)
    assert st == s2.S2ATTN_ERR_UNSUPPORTED
    assert b"static scratch" in lib.s2attn_last_error()
