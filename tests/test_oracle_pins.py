"""Pins for the fp64 oracle: checks against things other than the oracle itself.

* library special case: per head and group, torch.roll + torch's scaled_dot_product_attention
  (fp64, is_causal) and autograd through them must equal the oracle's forward and its
  hand-derived backward (LongLoRA summary page, §3.4 Algorithm 1 read with a library
  ``self_attn``);
* one group and no shift must be full causal attention (§3.4 "The core computational
  problem"; the inference-time full attention of §3 "LoRA+ ... full attention at inference");
* locality, including the page's worked example at N=8192, G=2048 (§3.4 "What the shift
  accomplishes operationally");
* direction invariance of the roll when G divides N (§3.4 "Why shifting direction doesn't
  matter", Table 8);
* the worked roll example (§3.4 "Step 2: Shift one chunk"), from tests/golden;
* Variant 2 of Table 8 (wrapped tokens in their own group): equal to the library version with
  the wrap group split by an explicit mask, and identical to the default outside that group;
* Variant 3 of Table 8 (wrapped tokens moved to the front of the last group): equal to causal
  attention in original token order under a same-shifted-group mask, written without any roll;
* G not dividing N (Table 7): the padded view equals a block-diagonal causal mask on the
  rolled sequence;
* RoPE with Position Interpolation: pair norms preserved, scores depend only on the position
  difference, the inverse undoes it, PI scale 1 is plain RoPE, and a hand-worked d = 4 case;
* central finite differences of the forward against the backward;
* closed-form sums implied by rows of P summing to one;
* planted mistakes in the oracle must fail these pins.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import s2attn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def make(B, Hq, Hkv, N, d, seed=0):
    return (rand((B, N, Hq, d), seed), rand((B, N, Hkv, d), seed + 1),
            rand((B, N, Hkv, d), seed + 2), rand((B, N, Hq, d), seed + 3))


# --------------------------------------------------------------------------------------
# Library implementation: torch.roll + SDPA per head and group, autograd for gradients.
# --------------------------------------------------------------------------------------
def torch_s2attn(q, k, v, G, scale, shb, shift, wrap_own_group=False):
    B, N, Hq, d = q.shape
    rep = Hq // k.shape[2]
    outs, lses = [], []
    for h in range(Hq):
        s = shift if h >= shb else 0
        qh = torch.roll(q[:, :, h], -s, dims=1).reshape(B, N // G, G, d)
        kh = torch.roll(k[:, :, h // rep], -s, dims=1).reshape(B, N // G, G, d)
        vh = torch.roll(v[:, :, h // rep], -s, dims=1).reshape(B, N // G, G, -1)
        mask = torch.ones(N // G, G, G, dtype=torch.bool).tril()
        if wrap_own_group and s > 0:
            side = torch.arange(G) >= G - s          # rows that hold wrapped tokens
            mask[-1] &= side[:, None] == side[None, :]
        oh = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=scale)
        scores = scale * qh @ kh.transpose(-1, -2)
        scores = scores.masked_fill(~mask, float("-inf"))
        lh = torch.logsumexp(scores, dim=-1)
        outs.append(torch.roll(oh.reshape(B, N, -1), s, dims=1))
        lses.append(torch.roll(lh.reshape(B, N), s, dims=1))
    return torch.stack(outs, dim=2), torch.stack(lses, dim=1)


def library_errors(B, Hq, Hkv, N, G, d, shb=None, shift=None, seed=0):
    """Max-abs differences (o, lse, dq, dk, dv) between the oracle and the library version."""
    q, k, v, do = make(B, Hq, Hkv, N, d, seed)
    scale = 1.0 / np.sqrt(d)
    shb_ = Hq // 2 if shb is None else shb
    shift_ = G // 2 if shift is None else shift
    o, lse = orc.s2attn_forward(q, k, v, G, scale, shb, shift)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale, shb, shift)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to, tl = torch_s2attn(tq, tk, tv, G, scale, shb_, shift_)
    to.backward(torch.tensor(do))
    return [float(np.abs(a - b.detach().numpy()).max()) for a, b in
            ((o, to), (lse, tl), (dq, tq.grad), (dk, tk.grad), (dv, tv.grad))]


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d", [
    (1, 4, 4, 64, 16, 8),       # multi-head, 4 groups
    (2, 4, 2, 48, 16, 8),       # GQA, 3 groups, batch 2
    (1, 8, 1, 32, 8, 4),        # MQA: every query head reads kv head 0 (mixed shifts)
    (1, 6, 3, 40, 8, 4),        # a GQA pair that straddles the head split (heads 2, 3)
])
def test_matches_library_attention(B, Hq, Hkv, N, G, d):
    errs = library_errors(B, Hq, Hkv, N, G, d)
    assert max(errs) < 1e-12, errs


@pytest.mark.parametrize("shb,shift", [(0, None), (4, None), (2, 24), (2, 8), (2, 0)])
def test_matches_library_patterns(shb, shift):
    # Pattern 2 only (all heads shifted), Pattern 1 only (none), shift up (roll +G/2,
    # written as shift = N - G/2), a different roll amount, and a zero roll.
    errs = library_errors(1, 4, 2, 32, 16, 4, shb=shb, shift=shift)
    assert max(errs) < 1e-12, errs


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d,shift", [(1, 4, 4, 64, 16, 8, 8), (2, 4, 2, 48, 16, 8, 4),
                                                  (1, 2, 1, 32, 32, 4, 16)])
def test_variant2_matches_library_with_split_mask(B, Hq, Hkv, N, G, d, shift):
    q, k, v, do = make(B, Hq, Hkv, N, d, 11)
    scale = 1.0 / np.sqrt(d)
    o, lse = orc.s2attn_forward(q, k, v, G, scale, None, shift, wrap_own_group=True)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale, None, shift, wrap_own_group=True)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to, tl = torch_s2attn(tq, tk, tv, G, scale, Hq // 2, shift, wrap_own_group=True)
    to.backward(torch.tensor(do))
    for a, b in ((o, to), (lse, tl), (dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(a - b.detach().numpy()).max() < 1e-12


def test_variant2_only_changes_the_wrap_group():
    """Unshifted heads and every shifted-head token outside the last rolled group are
    bit-identical to the default; the wrapped tokens (0..shift-1) see only each other."""
    B, Hq, N, G, d, shift = 1, 4, 64, 16, 8, 8
    q, k, v, do = make(B, Hq, Hq, N, d, 5)
    a, la = orc.s2attn_forward(q, k, v, G, 0.3, None, shift)
    b, lb = orc.s2attn_forward(q, k, v, G, 0.3, None, shift, wrap_own_group=True)
    assert np.array_equal(a[:, :, :2], b[:, :, :2])
    wrap_tokens = np.r_[N - (G - shift):N, 0:shift]
    keep = np.setdiff1d(np.arange(N), wrap_tokens)
    assert np.array_equal(a[:, keep, 2:], b[:, keep, 2:])
    assert not np.allclose(a[:, wrap_tokens, 2:], b[:, wrap_tokens, 2:])
    # tokens 0..shift-1 of a shifted head: plain causal attention over those tokens alone
    h = 3
    sq = 0.3 * q[0, :shift, h] @ k[0, :shift, h].T
    sq = np.where(np.tril(np.ones((shift, shift), dtype=bool)), sq, -np.inf)
    p = np.exp(sq - sq.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(b[0, :shift, h], p @ v[0, :shift, h], atol=1e-13)


def original_order_s2attn(q, k, v, G, scale, shb, shift):
    """Variant 3 written without any roll: in original token order, a shifted head attends
    causally (key not after query) within its shifted group, the group of token t being
    ((t - shift) mod N) // G; an unshifted head within t // G. torch SDPA with that mask."""
    B, N, Hq, d = q.shape
    rep = Hq // k.shape[2]
    t = torch.arange(N)
    outs, lses = [], []
    for h in range(Hq):
        s = shift if h >= shb else 0
        gid = ((t - s) % N) // G
        mask = (gid[:, None] == gid[None, :]) & (t[None, :] <= t[:, None])
        qh, kh, vh = q[:, :, h], k[:, :, h // rep], v[:, :, h // rep]
        outs.append(F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=scale))
        scores = (scale * qh @ kh.transpose(-1, -2)).masked_fill(~mask, float("-inf"))
        lses.append(torch.logsumexp(scores, dim=-1))
    return torch.stack(outs, dim=2), torch.stack(lses, dim=1)


def variant3_errors(B, Hq, Hkv, N, G, d, shift, seed=13):
    q, k, v, do = make(B, Hq, Hkv, N, d, seed)
    scale = 1.0 / np.sqrt(d)
    o, lse = orc.s2attn_forward(q, k, v, G, scale, None, shift, wrap_front_first=True)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale, None, shift, wrap_front_first=True)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to, tl = original_order_s2attn(tq, tk, tv, G, scale, Hq // 2, shift)
    to.backward(torch.tensor(do))
    return [float(np.abs(a - b.detach().numpy()).max()) for a, b in
            ((o, to), (lse, tl), (dq, tq.grad), (dk, tk.grad), (dv, tv.grad))]


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d,shift", [
    (1, 4, 4, 64, 16, 8, 8),     # half-group roll
    (2, 4, 2, 48, 16, 8, 4),     # GQA, batch 2, quarter-group roll
    (1, 8, 1, 32, 8, 4, 6),      # MQA, most of the group wrapped
])
def test_variant3_is_causal_in_original_order_within_shifted_groups(B, Hq, Hkv, N, G, d, shift):
    """Variant 3 (Table 8, Figure 6): with the wrapped tokens moved to the front of the last
    group, every group's causal order is the original token order, so the oracle's roll,
    group, swap, attend, unswap, unroll sequence must equal causal attention in original
    order under a same-shifted-group mask (no roll anywhere), forward, LSE and autograd."""
    assert max(variant3_errors(B, Hq, Hkv, N, G, d, shift)) < 1e-12


def test_variant3_against_default_and_variant2():
    """Outside the last rolled group Variant 3 is bit-identical to the default; the wrapped
    tokens see only each other (as in Variant 2); the other tokens of that group now also
    see the wrapped ones, which changes their outputs."""
    B, Hq, N, G, d, shift = 1, 4, 64, 16, 8, 8
    q, k, v, do = make(B, Hq, Hq, N, d, 5)
    a, _ = orc.s2attn_forward(q, k, v, G, 0.3, None, shift)
    b, _ = orc.s2attn_forward(q, k, v, G, 0.3, None, shift, wrap_own_group=True)
    c, _ = orc.s2attn_forward(q, k, v, G, 0.3, None, shift, wrap_front_first=True)
    assert np.array_equal(a[:, :, :2], c[:, :, :2])
    last = np.r_[N - (G - shift):N, 0:shift]
    keep = np.setdiff1d(np.arange(N), last)
    assert np.array_equal(a[:, keep, 2:], c[:, keep, 2:])
    np.testing.assert_allclose(c[:, :shift, 2:], b[:, :shift, 2:], atol=1e-13)
    back = np.arange(N - (G - shift), N)
    assert not np.allclose(c[:, back, 2:], a[:, back, 2:])


def _swap_never_undone(x, N, G, shb, shift, enabled, inverse=False):
    return _SWAP(x, N, G, shb, shift, enabled, inverse=False)


def test_planted_variant3_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "_swap_wrap_front", _swap_never_undone)
    # (with shift = G/2 a second forward swap would undo the first: use shift != G/2)
    assert max(variant3_errors(1, 4, 2, 32, 8, 4, 2, seed=3)) > 1e-3


def block_mask_s2attn(q, k, v, G, scale, shb, shift):
    """G not dividing N, written without the view into groups: per head, torch.roll, then
    SDPA over the whole rolled sequence with the mask 'same block of G rows (the last block
    shorter), key not after query', then the roll back."""
    B, N, Hq, d = q.shape
    rep = Hq // k.shape[2]
    r = torch.arange(N)
    mask = ((r[:, None] // G) == (r[None, :] // G)) & (r[None, :] <= r[:, None])
    outs, lses = [], []
    for h in range(Hq):
        s = shift if h >= shb else 0
        qh = torch.roll(q[:, :, h], -s, dims=1)
        kh = torch.roll(k[:, :, h // rep], -s, dims=1)
        vh = torch.roll(v[:, :, h // rep], -s, dims=1)
        oh = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask, scale=scale)
        scores = (scale * qh @ kh.transpose(-1, -2)).masked_fill(~mask, float("-inf"))
        outs.append(torch.roll(oh, s, dims=1))
        lses.append(torch.roll(torch.logsumexp(scores, dim=-1), s, dims=1))
    return torch.stack(outs, dim=2), torch.stack(lses, dim=1)


@pytest.mark.parametrize("B,Hq,Hkv,N,G,d,shift", [
    (1, 4, 4, 40, 16, 8, 8),     # two full groups and one of 8
    (2, 4, 2, 52, 24, 4, 12),    # GQA, batch 2, last group of 4
    (1, 2, 1, 20, 32, 4, 16),    # G > N: a single, partial group
])
def test_partial_last_group_matches_block_mask(B, Hq, Hkv, N, G, d, shift):
    """G not dividing N (Table 7's 1/6 group): the oracle's padding to a multiple of G equals
    attention under a block-diagonal causal mask on the rolled sequence, forward, LSE and
    autograd."""
    q, k, v, do = make(B, Hq, Hkv, N, d, 17)
    scale = 1.0 / np.sqrt(d)
    kw = dict(partial_last_group=True)
    o, lse = orc.s2attn_forward(q, k, v, G, scale, None, shift, **kw)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale, None, shift, **kw)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    to, tl = block_mask_s2attn(tq, tk, tv, G, scale, Hq // 2, shift)
    to.backward(torch.tensor(do))
    for a, b in ((o, to), (lse, tl), (dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.abs(a - b.detach().numpy()).max() < 1e-12


def test_partial_last_group_option_is_inert_when_g_divides_n():
    q, k, v, do = make(1, 4, 2, 48, 4, 19)
    a = orc.s2attn_forward(q, k, v, 16, 0.5, None, 8)
    b = orc.s2attn_forward(q, k, v, 16, 0.5, None, 8, partial_last_group=True)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    with pytest.raises(ValueError):
        orc.s2attn_forward(q[:, :40], k[:, :40], v[:, :40], 16, 0.5, None, 8)


def test_one_group_no_shift_is_full_causal_attention():
    B, Hq, N, d = 2, 3, 40, 8
    q, k, v, do = make(B, Hq, Hq, N, d, 7)
    scale = 0.3
    o, lse = orc.s2attn_forward(q, k, v, N, scale, shift_head_begin=Hq)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, N, scale, shift_head_begin=Hq)
    tq, tk, tv = (torch.tensor(x).transpose(1, 2).requires_grad_() for x in (q, k, v))
    to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True, scale=scale)
    to.backward(torch.tensor(do).transpose(1, 2))
    np.testing.assert_allclose(o, to.transpose(1, 2).detach().numpy(), atol=1e-13)
    for a, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(a, t.grad.transpose(1, 2).numpy(), atol=1e-12)
    s = scale * torch.tensor(q).transpose(1, 2) @ torch.tensor(k).transpose(1, 2).transpose(-1, -2)
    s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-13)


def test_worked_roll_example():
    ex = json.load(open(os.path.join(GOLDEN, "longlora_roll_example.json")))
    N, G, s = ex["N"], ex["G"], ex["shift"]
    tok = orc.rolled_token_index(N, G, s).reshape(-1)
    assert tok[0] + 1 == ex["roll_1based"]["token_at_position_1"]
    assert tok[1] + 1 == ex["roll_1based"]["token_at_position_2"]
    assert tok[0] == ex["roll_0based"]["token_at_rolled_position_0"]
    assert int(np.nonzero(tok == 0)[0][0]) == ex["roll_0based"]["rolled_position_of_token_0"]
    first = orc.rolled_token_index(N, G, s)[0]
    assert (first[0] + 1, first[-1] + 1) == tuple(ex["shifted_head_first_group_1based"])
    unshifted = orc.rolled_token_index(N, G, 0)[0]
    assert (unshifted[0] + 1, unshifted[-1] + 1) == tuple(ex["unshifted_first_group_1based"])
    lo, hi = ex["token_2048_1based"]["same_group_shifted_head_contains"]
    assert lo - 1 in first and hi - 1 in first
    assert ex["token_2048_1based"]["unshifted_group_excludes"] - 1 not in unshifted


def test_worked_example_locality_full_size():
    """N=8192, G=2048: which tokens can change token 2048's (1-based) output."""
    N, G, d = 8192, 2048, 4
    q, k, v, _ = make(1, 2, 2, N, d, 3)
    base, _ = orc.s2attn_forward(q, k, v, G, 0.5)
    t = 2047   # 0-based token 2048

    def changed(tok):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for x in (q2, k2, v2):
            x[0, tok] += 1.0
        o, _ = orc.s2attn_forward(q2, k2, v2, G, 0.5)
        return [bool(np.any(o[0, t, h] != base[0, t, h])) for h in (0, 1)]

    # [unshifted head 0, shifted head 1]
    assert changed(3072) == [False, False]   # 1-based 3073: outside both groups
    assert changed(2048) == [False, False]   # 1-based 2049: same shifted group, but later
    assert changed(1023) == [True, False]    # 1-based 1024: unshifted group only
    assert changed(1024) == [True, True]     # 1-based 1025: first token of the shifted group
    assert changed(0) == [True, False]


def test_locality_bitwise_small():
    B, Hq, N, G, d = 1, 4, 64, 16, 8
    q, k, v, do = make(B, Hq, Hq, N, d, 11)
    o0, l0 = orc.s2attn_forward(q, k, v, G, 0.35)
    dq0, dk0, dv0 = orc.s2attn_backward(q, k, v, do, G, 0.35)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for x in (q2, k2, v2):
        x[0, 40] += 3.0  # token 40: unshifted group 2 = [32, 48); shifted group [40, 56)
    o1, l1 = orc.s2attn_forward(q2, k2, v2, G, 0.35)
    dq1, dk1, dv1 = orc.s2attn_backward(q2, k2, v2, do, G, 0.35)
    unaffected_unshifted = [t for t in range(N) if not 32 <= t < 48]
    unaffected_shifted = [t for t in range(N) if not 40 <= t < 56]
    for a, b in ((o0, o1), (dq0, dq1), (dk0, dk1), (dv0, dv1)):
        assert np.array_equal(a[0, unaffected_unshifted, :2], b[0, unaffected_unshifted, :2])
        assert np.array_equal(a[0, unaffected_shifted, 2:], b[0, unaffected_shifted, 2:])
        assert not np.array_equal(a[0, 41, 2], b[0, 41, 2])
    assert np.array_equal(l0[0, :2, unaffected_unshifted], l1[0, :2, unaffected_unshifted])


def test_direction_invariance_exact():
    """Rolling by +G/2 instead of -G/2 forms the same groups when G divides N."""
    B, Hq, Hkv, N, G, d = 1, 4, 2, 96, 32, 8
    q, k, v, do = make(B, Hq, Hkv, N, d, 5)
    down = orc.s2attn_forward(q, k, v, G, 0.4, shift=G // 2)
    up = orc.s2attn_forward(q, k, v, G, 0.4, shift=N - G // 2)
    for a, b in zip(down, up):
        assert np.array_equal(a, b)
    gd = orc.s2attn_backward(q, k, v, do, G, 0.4, shift=G // 2)
    gu = orc.s2attn_backward(q, k, v, do, G, 0.4, shift=N - G // 2)
    for a, b in zip(gd, gu):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-15)


@pytest.mark.parametrize("Hkv", [4, 2])
def test_finite_differences(Hkv):
    B, Hq, N, G, d = 1, 4, 8, 4, 4
    q, k, v, do = make(B, Hq, Hkv, N, d, 21 + Hkv)
    scale = 0.45
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale)

    def loss(q_, k_, v_):
        return float((orc.s2attn_forward(q_, k_, v_, G, scale)[0] * do).sum())

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        args = [q, k, v]
        fd = np.zeros_like(args[which])
        it = np.nditer(args[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        rel = np.abs(fd - grad).max() / np.abs(grad).max()
        assert rel < 1e-6, (which, rel)


def test_closed_form_sums():
    B, Hq, N, G, d = 1, 4, 64, 16, 8
    q, k, v, do = make(B, Hq, Hq, N, d, 31)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, 0.3)
    for h in range(Hq):
        shift = G // 2 if h >= Hq // 2 else 0
        for toks in orc.rolled_token_index(N, G, shift):
            np.testing.assert_allclose(dv[0, toks, h].sum(0), do[0, toks, h].sum(0), atol=1e-12)
            np.testing.assert_allclose(dk[0, toks, h].sum(0), 0.0, atol=1e-12)
    o, _ = orc.s2attn_forward(q, k, v, G, 0.3)
    assert np.isfinite(o).all()


def test_head_group_rows_matches_full():
    """The row-restricted evaluation used at large sizes equals the full oracle."""
    B, Hq, Hkv, N, G, d = 1, 4, 2, 64, 32, 8
    q, k, v, do = make(B, Hq, Hkv, N, d, 41)
    scale = 0.33
    o, lse = orc.s2attn_forward(q, k, v, G, scale)
    dq, dk, dv = orc.s2attn_backward(q, k, v, do, G, scale)
    rep = Hq // Hkv
    for kvh in range(Hkv):
        acc = {}
        for h in range(kvh * rep, (kvh + 1) * rep):
            shift = G // 2 if h >= Hq // 2 else 0
            for g in range(N // G):
                r = orc.head_group_rows(q[0, :, h], k[0, :, kvh], v[0, :, kvh], do[0, :, h], G,
                                        scale, shift, g, [0, 5, G - 1], kv_rows=[3, 17, G - 1])
                np.testing.assert_allclose(r["o"], o[0, r["q_tok"], h], atol=1e-13)
                np.testing.assert_allclose(r["lse"], lse[0, h, r["q_tok"]], atol=1e-13)
                np.testing.assert_allclose(r["dq"], dq[0, r["q_tok"], h], atol=1e-13)
                for i, t in enumerate(r["kv_tok"]):
                    a = acc.setdefault(int(t), [0.0, 0.0])
                    a[0] = a[0] + r["dk"][i]
                    a[1] = a[1] + r["dv"][i]
        for t, (a_dk, a_dv) in acc.items():
            np.testing.assert_allclose(a_dk, dk[0, t, kvh], atol=1e-13)
            np.testing.assert_allclose(a_dv, dv[0, t, kvh], atol=1e-13)


# --------------------------------------------------------------------------------------
# Planted mistakes: each must be caught by one of the pins above.
# --------------------------------------------------------------------------------------
def _tile_kv(x, Hq):
    return np.tile(x, (1, 1, Hq // x.shape[2], 1))


_SWAP = orc._swap_wrap_front


def _leaky_probs(q, k, scale, split=None):
    G = q.shape[0]
    s = scale * (q @ k.T)
    s = np.where(np.tril(np.ones((G, G), dtype=bool), k=1), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def _backward_without_rowsum(q, k, v, do, scale, splits=None):
    Bg, G, H, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(Bg):
        for h in range(H):
            p, _ = orc._group_probs(q[b, :, h], k[b, :, h], scale)
            ds = p * (do[b, :, h] @ v[b, :, h].T)
            dq[b, :, h] = scale * (ds @ k[b, :, h])
            dk[b, :, h] = scale * (ds.T @ q[b, :, h])
            dv[b, :, h] = p.T @ do[b, :, h]
    return dq, dk, dv


def _roll_no_rollback(x, amount, shift_head_begin):
    out = x.copy()
    if amount < 0:
        out[:, :, shift_head_begin:] = np.roll(x[:, :, shift_head_begin:], amount, axis=1)
    return out


@pytest.mark.parametrize("name,target,mutant", [
    ("kv heads tiled instead of repeated", "expand_kv", _tile_kv),
    ("mask lets one future token through", "_group_probs", _leaky_probs),
    ("dS without the row-sum term", "causal_self_attn_backward", _backward_without_rowsum),
    ("output not rolled back", "chunk_roll", _roll_no_rollback),
])
def test_planted_mistakes_are_caught(monkeypatch, name, target, mutant):
    monkeypatch.setattr(orc, target, mutant)
    errs = library_errors(1, 4, 2, 32, 8, 4, seed=3)
    assert max(errs) > 1e-3, (name, errs)


# --------------------------------------------------------------------------------------
# RoPE with Position Interpolation (the step before the attention)
# --------------------------------------------------------------------------------------
def test_rope_preserves_pair_norms_and_inverts():
    x = rand((2, 9, 3, 8), 41)
    y = orc.rope_pi(x, pi_scale=0.5)
    n = lambda a: a[..., :4] ** 2 + a[..., 4:] ** 2
    np.testing.assert_allclose(n(y), n(x), rtol=1e-13)
    np.testing.assert_allclose(orc.rope_pi(y, pi_scale=0.5, inverse=True), x, atol=1e-13)
    assert np.array_equal(orc.rope_pi(x[:, :1]), x[:, :1])          # token 0: no rotation


def test_rope_scores_depend_only_on_the_offset():
    """The defining property of rotary embeddings: <R(m) q, R(n) k> = <R(m + c) q, R(n + c) k>.
    Checked by placing the same q and k at positions shifted by c."""
    d, N, c = 16, 12, 5
    q, k = rand((d,), 1), rand((d,), 2)
    x = np.zeros((1, N + c, 2, d))
    x[0, 3, 0], x[0, 7, 1] = q, k              # q at 3, k at 7
    x[0, 3 + c, 0], x[0, 7 + c, 1] = q, k      # the same pair shifted by c
    y = orc.rope_pi(x, base=100.0, pi_scale=0.75)
    a = y[0, 3, 0] @ y[0, 7, 1]
    b = y[0, 3 + c, 0] @ y[0, 7 + c, 1]
    assert abs(a - b) < 1e-12


def test_rope_position_interpolation_is_a_position_rescale():
    """Position Interpolation with scale 1/2: token t turns as far as token t/2 would without
    it. Checked by placing token t at position 2t and rotating with scale 1/2."""
    x = rand((1, 16, 2, 8), 43)
    w = np.zeros((1, 32, 2, 8))
    w[:, ::2] = x
    np.testing.assert_allclose(orc.rope_pi(w, pi_scale=0.5)[:, ::2], orc.rope_pi(x), atol=1e-13)


def test_rope_hand_worked_case():
    """d = 4, base 100: theta = (1, 1/10). Token 2 with PI scale 1/2 sits at position 1:
    pair 0 (x0, x2) turns by 1 rad, pair 1 (x1, x3) by 0.1 rad."""
    x = np.zeros((1, 3, 1, 4))
    x[0, 2, 0] = [1.0, 2.0, 3.0, 4.0]
    y = orc.rope_pi(x, base=100.0, pi_scale=0.5)[0, 2, 0]
    c1, s1, c2, s2 = np.cos(1.0), np.sin(1.0), np.cos(0.1), np.sin(0.1)
    want = [1 * c1 - 3 * s1, 2 * c2 - 4 * s2, 3 * c1 + 1 * s1, 4 * c2 + 2 * s2]
    np.testing.assert_allclose(y, want, atol=1e-15)
