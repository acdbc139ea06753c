"""Variant 2 of the S²-Attn ablation (LongLoRA summary page, §3.4 "Information leakage
considerations", Table 8 and Figure 6): in the rolled heads the tokens that the roll wrapped
around form their own causal group. CUDA path (S2ATTN_FLAG_WRAP_OWN_GROUP) against the oracle
(wrap_own_group=True), element by element.
"""
import zlib

import numpy as np
import pytest
import torch

import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200.inputs import make_inputs

from gpu_helpers import check_case, gpu_run

pytestmark = pytest.mark.gpu
V2 = s2.S2ATTN_FLAG_WRAP_OWN_GROUP


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.lib()


@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shb,shift", [
    # the default half-group roll: the wrapped half group and the last half group split
    ("half", 1, 4, 4, 512, 128, 128, None, None),
    # the split falls inside a 128-row tile (shift 32), GQA, ragged tail, batch 2
    ("ragged_gqa", 2, 4, 2, 320, 64, 64, None, None),
    # groups straddle tiles, split mid-tile
    ("straddle", 1, 4, 4, 384, 192, 128, None, 96),
    # several tiles per group, split on a tile edge (triangular dS packing is off)
    ("aligned", 1, 8, 4, 2048, 512, 128, None, None),
    # every head rolled, MQA
    ("pattern2_mqa", 1, 8, 1, 512, 128, 128, 0, 40),
    # a small wrap remainder (shift 8) and a large one (G - 8)
    ("shift8", 1, 2, 2, 256, 128, 64, None, 8),
    ("shift_g_minus_8", 1, 2, 2, 256, 128, 64, None, 120),
])
def test_variant2_matches_oracle(name, B, Hq, Hkv, N, G, d, shb, shift):
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32(("v2" + name).encode()) % 10000, shb=shb,
               shift=shift, flags=V2)


@pytest.mark.parametrize("mode", ["recompute", "per_kv_head"])
def test_variant2_backward_paths(mode):
    check_case(1, 8, 4, 1024, 256, 128, seed=77, flags=V2, mode=mode)


def test_variant2_touches_only_the_last_rolled_group():
    """Outside the last group of the rolled heads the two variants compute the same rows, so
    the kernels must agree bit for bit there (same tiles, same order)."""
    B, Hq, Hkv, N, G, d = 1, 4, 4, 512, 128, 64
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, 5, 1.0)
    scale = d ** -0.5
    a = gpu_run(q, k, v, do, G, scale, backward=False)
    b = gpu_run(q, k, v, do, G, scale, backward=False, flags=V2)
    shb, sh = Hq // 2, G // 2
    # rolled row r holds original token (r + sh) mod N; the last rolled group is rows N-G..N-1
    last = (np.arange(N - G, N) + sh) % N
    keep = np.setdiff1d(np.arange(N), last)
    assert torch.equal(a["o"][:, :, :shb], b["o"][:, :, :shb])
    assert torch.equal(a["o"][:, keep, shb:], b["o"][:, keep, shb:])
    assert not torch.equal(a["o"][:, last, shb:], b["o"][:, last, shb:])
