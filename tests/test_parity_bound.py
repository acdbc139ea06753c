"""The GPU tests' bf16 bound, checked on the CPU: the half-ulp term u(x) is exactly the most
that rounding to bf16 can move a value, and no more."""
import numpy as np
import torch

from gpu_helpers import bf16_half_ulp


def test_half_ulp_bounds_bf16_rounding_tightly():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, s, 20000) for s in (1e-3, 1.0, 10.0, 300.0)])
    r = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    u = bf16_half_ulp(r)
    assert (np.abs(r - x) <= u).all()
    # a value halfway between two bf16 neighbours is moved by exactly u
    assert bf16_half_ulp(np.array([1.0, 1.5, 2.0, 8.0, 12.0, -3.0])).tolist() == \
        [2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -5, 2.0 ** -5, 2.0 ** -7]
    mid = np.float64(1.0 + 2.0 ** -8)          # halfway between 1 and 1 + 2^-7
    assert abs(float(torch.tensor(mid).to(torch.bfloat16)) - mid) == 2.0 ** -8
    assert bf16_half_ulp(np.array([0.0]))[0] == 0.0
