"""Variants 2 and 3 of the S²-Attn ablation, and groups that do not divide the sequence (LongLoRA summary page, §3.4 "Information leakage
considerations", Table 8 and Figure 6). Variant 2: in the rolled heads the tokens that the roll
wrapped around form their own causal group (S2ATTN_FLAG_WRAP_OWN_GROUP, oracle
wrap_own_group=True). Variant 3: they move to the front of the last group, so its causal order
is the original token order (S2ATTN_FLAG_WRAP_FRONT_FIRST, oracle wrap_front_first=True).
G not dividing N (Table 7's 1/6 group): S2ATTN_FLAG_PARTIAL_LAST_GROUP, the last rolled group
shorter (oracle partial_last_group=True).
CUDA path against the oracle, element by element.
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
V3 = s2.S2ATTN_FLAG_WRAP_FRONT_FIRST
PARTIAL = s2.S2ATTN_FLAG_PARTIAL_LAST_GROUP


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.lib()


SHAPES = [
    # the default half-group roll
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
    # Variant 3: a rolled tile made of three runs of tokens (rows 128..191 -> 144..207,
    # 192..207 -> 0..15, 208..255 -> 208..255)
    ("three_runs", 1, 2, 2, 256, 64, 64, None, 16),
    # one group: Variant 3 reorders the whole sequence back into plain causal order
    ("one_group", 1, 2, 2, 384, 384, 64, None, 136),
]


@pytest.mark.parametrize("flags", [V2, V3], ids=["variant2", "variant3"])
@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shb,shift", SHAPES)
def test_variant_matches_oracle(flags, name, B, Hq, Hkv, N, G, d, shb, shift):
    variant = 2 if flags == V2 else 3
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32(("v%d" % variant + name).encode()) % 10000,
               shb=shb, shift=shift, flags=flags)


@pytest.mark.parametrize("flags", [V2, V3], ids=["variant2", "variant3"])
@pytest.mark.parametrize("mode", ["recompute", "per_kv_head", "phases"])
def test_variant_backward_paths(flags, mode):
    check_case(1, 8, 4, 1024, 256, 128, seed=77 + flags, flags=flags, mode=mode)


@pytest.mark.parametrize("flags", [V2, V3], ids=["variant2", "variant3"])
def test_variant_touches_only_the_last_rolled_group(flags):
    """Outside the last group of the rolled heads the variants compute the same rows as the
    default, so the kernels must agree bit for bit there (same tiles, same order)."""
    B, Hq, Hkv, N, G, d = 1, 4, 4, 512, 128, 64
    q, k, v, do = make_inputs(B, Hq, Hkv, N, d, 5, 1.0)
    scale = d ** -0.5
    a = gpu_run(q, k, v, do, G, scale, backward=False)
    b = gpu_run(q, k, v, do, G, scale, backward=False, flags=flags)
    shb, sh = Hq // 2, G // 2
    # rolled row r holds original token (r + sh) mod N; the last rolled group is rows N-G..N-1
    last = (np.arange(N - G, N) + sh) % N
    keep = np.setdiff1d(np.arange(N), last)
    assert torch.equal(a["o"][:, :, :shb], b["o"][:, :, :shb])
    assert torch.equal(a["o"][:, keep, shb:], b["o"][:, keep, shb:])
    assert not torch.equal(a["o"][:, last, shb:], b["o"][:, last, shb:])


@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shb,shift", [
    # two full groups of one tile and a half-tile group; GQA
    ("tail_half_tile", 1, 4, 2, 320, 128, 64, None, None),
    # G > N: one partial group, rolled
    ("g_exceeds_n", 1, 2, 2, 72, 128, 64, None, None),
    # groups that straddle tiles, a ragged sequence, batch 2
    ("straddle_ragged", 2, 4, 4, 1000, 96, 128, None, None),
    # the metric shape's group with a sequence of 4.3 groups
    ("long_tail", 1, 2, 2, 8832, 2048, 128, None, None),
])
def test_partial_last_group_matches_oracle(name, B, Hq, Hkv, N, G, d, shb, shift):
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32(("partial" + name).encode()) % 10000,
               shb=shb, shift=shift, flags=PARTIAL)


@pytest.mark.parametrize("mode", ["recompute", "per_kv_head", "phases"])
def test_partial_last_group_backward_paths(mode):
    check_case(1, 4, 2, 704, 256, 128, seed=91, flags=PARTIAL, mode=mode)


# Groups and rolls that are not multiples of 8 rows: the remap's runs then start or end inside
# the 8-row atoms that TMA moves, and the kernels load those rows with plain loads.
ODD_SHAPES = [
    # the pages' group of 1/6 of the context (Table 7, "Group size ablation") at the metric
    # length: G = 1365, rolled by 682; the last rolled group has the 2 leftover rows
    ("table7_one_sixth", 1, 8, 4, 8192, 1365, 128, 682, PARTIAL),
    # odd G and roll, G | N
    ("odd_g", 1, 4, 4, 300, 75, 64, 37, 0),
    # odd G, shorter last group, two query heads per kv head
    ("odd_g_partial", 1, 4, 2, 1000, 333, 64, 166, PARTIAL),
    # N, G and roll all odd, batch 2
    ("all_odd", 2, 2, 2, 129, 43, 64, 21, 0),
    # Variants 2 and 3 with odd G and roll
    ("odd_g_variant2", 1, 4, 4, 693, 231, 64, 115, V2),
    ("odd_g_variant3", 1, 4, 4, 693, 231, 64, 115, V3),
    # a roll of 37 with Variant 3: the last group's three runs all end inside atoms
    ("roll37_variant3", 1, 4, 2, 512, 128, 128, 37, V3),
]


@pytest.mark.parametrize("name,B,Hq,Hkv,N,G,d,shift,flags", ODD_SHAPES)
def test_any_group_and_roll_matches_oracle(name, B, Hq, Hkv, N, G, d, shift, flags):
    check_case(B, Hq, Hkv, N, G, d, seed=zlib.crc32(("odd" + name).encode()) % 10000,
               shift=shift, flags=flags)


@pytest.mark.parametrize("mode", ["recompute", "per_kv_head", "phases"])
def test_any_group_and_roll_backward_paths(mode):
    check_case(1, 4, 2, 1000, 333, 64, seed=123, shift=166, flags=PARTIAL, mode=mode)


def test_odd_group_default_roll():
    """The default entry points with an odd G roll the second half of the heads by
    floor(G / 2), as the oracle does."""
    check_case(1, 4, 4, 450, 75, 128, seed=9)
