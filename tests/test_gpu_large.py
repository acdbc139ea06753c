"""CUDA path vs the fp64 oracle at the full workload sizes, in the launch configuration the
bench times (the public fwd + bwd calls).

* Llama2-7B layer at N=8192, G=2048 (the metric workload): every element of O, LSE, dQ, dK,
  dV against the full oracle.
* N=32768/G=8192, B=4 at N=8192, N=102400/G=25600, and the Llama2-70B GQA shape: sampled
  (batch, head, group) units — heads {0, Hq/2-1, Hq/2, Hq-1} (for GQA: every query head of
  kv heads 0 and Hkv-1, so dK/dV sums are complete), groups {0, last (the wrap group of the
  rolled heads)} — each checked on sampled rows with the oracle's row-restricted evaluation:
  query rows (O, LSE, dQ) at the start, end and random places of the group; kv rows (dK, dV)
  at the end of the group, and at its start when G <= 8192.
"""
import numpy as np
import pytest
import torch

from oracle import s2attn_oracle as orc
from shifted_sparse_attention_fwd_b200.inputs import WORKLOADS, make_inputs, make_workload_inputs, to_f64

from gpu_helpers import assert_close, check_case, gpu_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_metric_workload_full():
    w = WORKLOADS["llama7b_n8192_g2048"]
    check_case(w.B, w.Hq, w.Hkv, w.N, w.G, w.d, w.seed)


@pytest.mark.parametrize("name", ["llama7b_n32768_g8192", "llama7b_b4_n8192_g2048",
                                  "llama70b_gqa_n32768_g8192", "llama7b_n102400_g25600"])
def test_full_size_sampled(name):
    w = WORKLOADS[name]
    q, k, v, do = make_workload_inputs(w)
    g = gpu_run(q, k, v, do, w.G, w.scale)
    rep = w.Hq // w.Hkv
    ng = w.N // w.G
    rng = np.random.default_rng(w.seed)
    if rep == 1:
        kv_heads = sorted({0, w.Hq // 2 - 1, w.Hq // 2, w.Hq - 1})
    else:
        kv_heads = [0, w.Hkv - 1]
    q_rows = np.unique(np.concatenate([np.arange(128), np.arange(w.G - 128, w.G),
                                       rng.integers(0, w.G, 64)]))
    kv_rows = np.arange(w.G - 256, w.G)
    if w.G <= 8192:
        kv_rows = np.concatenate([np.arange(8), kv_rows])
    for b in sorted({0, w.B - 1}):
        for kvh in kv_heads:
            acc = {}
            for h in range(kvh * rep, (kvh + 1) * rep):
                shift = w.G // 2 if h >= w.Hq // 2 else 0
                for gi in sorted({0, ng - 1}):
                    r = orc.head_group_rows(to_f64(q[b, :, h]), to_f64(k[b, :, kvh]),
                                            to_f64(v[b, :, kvh]), to_f64(do[b, :, h]), w.G,
                                            w.scale, shift, gi, q_rows, kv_rows)
                    t = r["q_tok"]
                    assert_close("o", g["o"][b, t, h], r["o"])
                    assert_close("lse", g["lse"][b, h, t], r["lse"])
                    assert_close("dq", g["dq"][b, t, h], r["dq"])
                    for i, tk in enumerate(r["kv_tok"]):
                        a = acc.setdefault(int(tk), [0.0, 0.0])
                        a[0] = a[0] + r["dk"][i]
                        a[1] = a[1] + r["dv"][i]
            # dK/dV rows that received every query head's contribution from sampled groups:
            # with all heads of the kv head rolled alike, a kv row's group is the same in each.
            toks = sorted(acc)
            dk_ref = np.stack([acc[t][0] for t in toks])
            dv_ref = np.stack([acc[t][1] for t in toks])
            assert_close("dk", g["dk"][b, toks, kvh], dk_ref)
            assert_close("dv", g["dv"][b, toks, kvh], dv_ref)


def test_full_causal_n8192_sampled():
    """Full causal attention (the pages' Phase 2: standard attention after fine-tuning) at the
    metric length through the same kernels: one group of G = N = 8192 rows and no rolled head.
    Every head on sampled rows against the oracle's row-restricted evaluation: query rows at
    the start, the end and random places of the sequence; kv rows at the start (seen by all
    8192 query rows) and at the end."""
    B, Hq, Hkv, N, d = 1, 8, 8, 8192, 128
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, 1006)
    scale = d ** -0.5
    g = gpu_run(q, k, v, do, N, scale, shb=Hq, shift=0)
    rng = np.random.default_rng(1006)
    q_rows = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N), rng.integers(0, N, 64)]))
    kv_rows = np.concatenate([np.arange(8), np.arange(N - 128, N)])
    for h in range(Hq):
        r = orc.head_group_rows(to_f64(q[0, :, h]), to_f64(k[0, :, h]), to_f64(v[0, :, h]),
                                to_f64(do[0, :, h]), N, scale, 0, 0, q_rows, kv_rows)
        t = r["q_tok"]
        assert_close("o", g["o"][0, t, h], r["o"])
        assert_close("lse", g["lse"][0, h, t], r["lse"])
        assert_close("dq", g["dq"][0, t, h], r["dq"])
        tk = r["kv_tok"]
        assert_close("dk", g["dk"][0, tk, h], r["dk"])
        assert_close("dv", g["dv"][0, tk, h], r["dv"])
