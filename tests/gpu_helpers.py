"""Helpers shared by the GPU tests: run the CUDA path through the C ABI, run the oracle on
the same seeded inputs, compare with the stated tolerances.

Tolerances: O, dQ, dK, dV (bf16) within max-abs 2e-2 and mean-abs 2e-3 of the fp64 oracle;
LSE (fp32) within max-abs 1e-4.

Reading of the bf16 max-abs bound: 2e-2 is the budget for the kernels' arithmetic; the
final rounding of each result to bf16 comes on top of it, so an element passes when
|gpu - ref| <= 2e-2 + u(gpu), u(x) = half a bf16 ulp at x (2^(e-8) for 2^e <= |x| < 2^(e+1)),
the most that rounding the exact kernel result to bf16 can move it. Without that term no bf16
value above 8 in magnitude (u = 2^-5 > 2e-2) could pass, and dK/dV summed over grouped-query
heads reach that. The mean-abs bound is applied as stated. Every comparison also records the
strict figures — max-abs, mean-abs, and how many elements exceed 2e-2 and so needed the u term —
and, when S2ATTN_PARITY_LOG names a file, appends them to it as one JSON line per case.
"""
import json
import os

import numpy as np
import torch

from oracle import s2attn_oracle as orc
import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import make_inputs, to_f64

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-4


def _bwd(qd, kd, vd, o, lse, dod, G, scale, shb, shift, mode, flags=0):
    """Backward through one of the library's paths:
    auto        the allocating convenience (dS hand-off, all kv heads in one pass when the
                default cap allows);
    recompute   the minimum workspace: the dQ kernel recomputes S and dP;
    per_kv_head room for one kv head's dS tiles: one dK/dV + dQ pass per kv head;
    phases      preprocess, s2attn_bwd_dkdv_ds and s2attn_bwd_dq_ds called one by one (their
                _general forms when flags are given)."""
    if mode == "auto":
        return s2.bwd(qd, kd, vd, o, lse, dod, G, scale, shb, shift, flags=flags)
    B, N, Hq, d = qd.shape
    Hkv = kd.shape[2]
    shb_ = Hq // 2 if shb is None else shb
    sh_ = G // 2 if shift is None else shift
    if mode == "recompute":
        n = s2.s2attn_bwd_workspace_size(B, Hq, N)
    else:
        n = s2.s2attn_bwd_workspace_size_ex(B, Hq, Hkv, N, d, G, shb_, sh_,
                                            1 if mode == "per_kv_head" else 0, flags)
    ws = torch.empty(n, dtype=torch.uint8, device=qd.device)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    if mode == "phases":
        s2.s2attn_bwd_preprocess(o, lse, dod, ws)
        s2.s2attn_bwd_dkdv_ds(qd, kd, vd, dod, dk, dv, G, ws, scale, shb_, sh_, flags=flags)
        s2.s2attn_bwd_dq_ds(kd, dq, G, ws, scale, shb_, sh_, flags=flags)
    else:
        s2.s2attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, G, scale, shb_, sh_, ws, flags=flags)
    return dq, dk, dv


def gpu_run(q, k, v, do, G, scale, shb=None, shift=None, backward=True, mode="auto", flags=0):
    """Forward (+ backward) of the CUDA path on bf16 CPU inputs; returns CPU tensors."""
    dev = torch.device("cuda")
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o, lse = s2.fwd(qd, kd, vd, G, scale, shb, shift, flags=flags)
    out = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = _bwd(qd, kd, vd, o, lse, dod, G, scale, shb, shift, mode, flags)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    st, code = s2.s2attn_get_device_error()
    assert st == s2.S2ATTN_OK, f"device error status {st} code {code:#x}"
    return {k_: v_.cpu() for k_, v_ in out.items()}


def oracle_run(q, k, v, do, G, scale, shb=None, shift=None, backward=True, flags=0):
    qf, kf, vf, dof = (to_f64(x) for x in (q, k, v, do))
    wrap = bool(flags & s2.S2ATTN_FLAG_WRAP_OWN_GROUP)
    front = bool(flags & s2.S2ATTN_FLAG_WRAP_FRONT_FIRST)
    partial = bool(flags & s2.S2ATTN_FLAG_PARTIAL_LAST_GROUP)
    kw = dict(wrap_own_group=wrap, wrap_front_first=front, partial_last_group=partial)
    o, lse = orc.s2attn_forward(qf, kf, vf, G, scale, shb, shift, **kw)
    out = {"o": o, "lse": lse}
    if backward:
        dq, dk, dv = orc.s2attn_backward(qf, kf, vf, dof, G, scale, shb, shift, **kw)
        out.update(dq=dq, dk=dk, dv=dv)
    return out


def bf16_half_ulp(x):
    """Half a bf16 ulp at each value of x: the largest move that rounding an exact value to
    bf16 (8 significant bits) can make, 2^(e-8) for 2^e <= |x| < 2^(e+1); 0 at x = 0."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(a)                      # a = m * 2^e, 0.5 <= m < 1
    return np.where(a > 0, np.ldexp(1.0, e - 9), 0.0)


def assert_close(name, gpu, ref):
    """Compare one output with the oracle; returns the strict figures of the comparison."""
    g = gpu.to(torch.float64).numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    ref = np.asarray(ref)
    d = np.abs(g - ref)
    mx, mean = float(d.max()), float(d.mean())
    assert np.isfinite(g).all(), f"{name}: non-finite output"
    rep = {"max_abs": mx, "mean_abs": mean, "n": int(d.size)}
    if name == "lse":
        assert mx <= LSE_MAX_ABS, f"lse max-abs {mx:.3g} > {LSE_MAX_ABS}"
        return rep
    over = d > BF16_MAX_ABS
    excess = float((d - BF16_MAX_ABS - bf16_half_ulp(g)).max())
    rep.update(n_over_2e2=int(over.sum()),
               max_abs_ref_where_over=float(np.abs(ref[over]).max()) if over.any() else 0.0,
               excess_over_bound=excess)
    assert excess <= 0, (f"{name} max-abs {mx:.3g} exceeds 2e-2 + half a bf16 ulp by {excess:.3g} "
                         f"(mean {mean:.3g})")
    assert mean <= BF16_MEAN_ABS, f"{name} mean-abs {mean:.3g} > {BF16_MEAN_ABS}"
    return rep


def log_case(case, report):
    """Append the strict figures of one case to the file S2ATTN_PARITY_LOG names, if any."""
    path = os.environ.get("S2ATTN_PARITY_LOG")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"case": case, **report}) + "\n")


def check_case(B, Hq, Hkv, N, G, d, seed, shb=None, shift=None, q_gain=1.0, scale=None,
               backward=True, mode="auto", flags=0, case=None):
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, seed, q_gain)
    scale = d ** -0.5 if scale is None else scale
    g = gpu_run(q, k, v, do, G, scale, shb, shift, backward, mode, flags)
    r = oracle_run(q, k, v, do, G, scale, shb, shift, backward, flags)
    report, failures = {}, []
    for name in g:
        try:
            report[name] = assert_close(name, g[name], r[name])
        except AssertionError as e:    # record every tensor's figures before failing
            failures.append(str(e))
            gg = g[name].to(torch.float64).numpy()
            report[name] = {"max_abs": float(np.abs(gg - r[name]).max()), "failed": str(e)}
    log_case(case or dict(B=B, Hq=Hq, Hkv=Hkv, N=N, G=G, d=d, seed=seed, shb=shb,
                          shift=shift, q_gain=q_gain, mode=mode, flags=flags), report)
    assert not failures, "; ".join(failures)
    return report
