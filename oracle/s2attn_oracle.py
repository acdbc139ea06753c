"""fp64 CPU oracle for S²-Attn (shifted sparse attention), forward and backward.

TEST INFRASTRUCTURE. This module exists to check the CUDA path. Only the test suite,
the smoke check and the bench's CPU-baseline leg may import or run it; the library
never calls it and has no CPU fallback.

Source: "LongLoRA: Efficient Fine-tuning of Long-Context Large Language Models",
paper-graph summary page, §3.4 "S2-Attn: Shifted Sparse Attention as a Training-Time
Proxy for Full Attention", Algorithm 1 (the roll, standard self-attention, the roll back)
and the three-step description (split heads, shift one chunk, recombine).

The forward is the algorithm written out literally, in the pages' notation:
  1. split the H heads into two chunks; roll the second chunk by -G/2 along N
     (``np.roll``, i.e. torch.roll semantics: rolled[r] = x[(r + G/2) mod N]);
  2. view the sequence as B*N/G independent groups of G tokens;
  3. run standard causal self-attention softmax(scale * q k^T) v inside each group;
  4. reshape back to [B, N, H, d] and roll the second chunk back by +G/2.
The backward differentiates those four steps directly: per group
dP = dO V^T, dS = P o (dP - rowsum(P o dP)), dQ = scale dS K, dK = scale dS^T Q,
dV = P^T dO; the derivative of a roll is the opposite roll and the derivative of the
shared K/V view (grouped-query heads) is a sum over the query heads that share it.

Readings where the page is silent:
  * scale: the page writes softmax(q k^T); the caller's ``scale`` multiplies q k^T.
  * causal mask: applied in rolled order within each group, so in the shifted heads the
    wrap group (last G/2 tokens followed by the first G/2) lets the first G/2 tokens see
    the last G/2 ones (the page's §3.4 "Information leakage considerations" accepts it).
  * LSE: natural log of the row sum of exp(scale * q k^T) over the allowed keys, stored
    per original token as [B, Hq, N].
  * grouped-query heads: query head h reads key/value head h // (Hq / Hkv); the shift of
    query head h is applied to that shared view.
  * ``shift_head_begin`` (default Hq/2, the page's chunk(2)) and ``shift`` (default G/2)
    generalise the split point and the roll amount for the ablation patterns; the roll
    is always rolled[r] = x[(r + shift) mod N].
  * ``wrap_own_group`` is the page's Variant 2 (Table 8, Figure 6): in the shifted heads the
    tokens that the roll wrapped around (original tokens 0..shift-1, the last ``shift``
    rolled rows) form their own group instead of sharing the last group with the last
    G - shift tokens; that last group is split at the wrap point into two causal groups.
  * ``wrap_front_first`` is the page's Variant 3 (Table 8, Figure 6): in the shifted heads
    the wrapped tokens swap places with the front of the last group, i.e. that group lists
    original tokens 0..shift-1 first and the last G - shift tokens after them, so its causal
    order is the original token order; every other group is unchanged.
  * ``partial_last_group`` admits N not divisible by G (Table 7 uses a group of 1/6 of the
    context): the rolled sequence is cut into groups of G rows with the last one shorter
    (N mod G rows). Done literally by padding: the rolled tensors are extended with zero rows to
    a multiple of G before the view into groups, and the pad rows' outputs are dropped. Pad rows
    come last in their group, so the causal mask keeps every real query away from them, and in
    the backward their upstream gradient is zero, so they contribute nothing.

Everything is float64; inputs are the bf16 values widened exactly.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "chunk_roll",
    "expand_kv",
    "causal_self_attn",
    "causal_self_attn_backward",
    "s2attn_forward",
    "s2attn_backward",
    "rolled_token_index",
    "head_group_rows",
    "rope_pi",
]


def chunk_roll(x: np.ndarray, amount: int, shift_head_begin: int) -> np.ndarray:
    """Roll heads [shift_head_begin, H) of x [B, N, H, ...] by ``amount`` along N.

    Algorithm 1 rolls with chunk_roll(qkv, -G/2, H/2) before the attention and back with
    chunk_roll(out, +G/2, H/2) after it. np.roll has torch.roll's semantics:
    np.roll(x, a)[r] = x[(r - a) mod N].
    """
    out = x.copy()
    out[:, :, shift_head_begin:] = np.roll(x[:, :, shift_head_begin:], amount, axis=1)
    return out


def expand_kv(x: np.ndarray, Hq: int) -> np.ndarray:
    """Per-query-head view of grouped key/value heads: head h reads kv head h // (Hq/Hkv)."""
    rep = Hq // x.shape[2]
    return np.repeat(x, rep, axis=2)


def _group_probs(q: np.ndarray, k: np.ndarray, scale: float, split: int | None = None):
    """Causal softmax of scale * q k^T for one group and head; q, k are [G, d].

    With ``split``, rows [0, split) and [split, G) are two separate causal groups.
    Returns (P, lse) with P [G, G] (zero above the diagonal) and lse [G].
    """
    G = q.shape[0]
    s = scale * (q @ k.T)
    allowed = np.tril(np.ones((G, G), dtype=bool))
    if split is not None:
        side = np.arange(G) >= split
        allowed &= side[:, None] == side[None, :]
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def causal_self_attn(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float, splits=None):
    """Standard causal self-attention on every batch element: q, k, v [Bg, G, H, d].

    This is the ``self_attn(qkv)`` call of Algorithm 1 after the view into groups.
    ``splits(bg, h)`` optionally names a row where group bg of head h splits in two.
    Returns o [Bg, G, H, d] and lse [Bg, G, H].
    """
    Bg, G, H, d = q.shape
    o = np.empty((Bg, G, H, v.shape[3]))
    lse = np.empty((Bg, G, H))
    for b in range(Bg):
        for h in range(H):
            sp = splits(b, h) if splits else None
            p, lse[b, :, h] = _group_probs(q[b, :, h], k[b, :, h], scale, sp)
            o[b, :, h] = p @ v[b, :, h]
    return o, lse


def causal_self_attn_backward(q, k, v, do, scale, splits=None):
    """Gradients of causal_self_attn for upstream do [Bg, G, H, d] (direct differentiation).

    Returns dq, dk, dv, each [Bg, G, H, d]; dk and dv are per query head (not yet summed
    over heads that share a kv head).
    """
    Bg, G, H, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for b in range(Bg):
        for h in range(H):
            sp = splits(b, h) if splits else None
            p, _ = _group_probs(q[b, :, h], k[b, :, h], scale, sp)
            dp = do[b, :, h] @ v[b, :, h].T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, :, h] = scale * (ds @ k[b, :, h])
            dk[b, :, h] = scale * (ds.T @ q[b, :, h])
            dv[b, :, h] = p.T @ do[b, :, h]
    return dq, dk, dv


def _defaults(Hq, G, shift_head_begin, shift):
    if shift_head_begin is None:
        shift_head_begin = Hq // 2
    if shift is None:
        shift = G // 2
    return shift_head_begin, shift


def _wrap_splits(B, N, G, shb, shift, wrap_own_group):
    """Variant 2: the last group of every batch element, in heads >= shb, splits at the wrap
    (in-group row G - shift: rolled rows N - shift .. N - 1 hold original tokens 0..shift-1)."""
    if not wrap_own_group:
        return None
    if not 0 < shift < G:
        raise ValueError("the wrap group exists for 0 < shift < G")
    ng = N // G
    return lambda bg, h: (G - shift) if (h >= shb and bg % ng == ng - 1) else None


def _swap_wrap_front(x: np.ndarray, N: int, G: int, shb: int, shift: int, enabled: bool,
                     inverse: bool = False) -> np.ndarray:
    """Variant 3 on the grouped view x [B*N/G, G, H, ...]: in heads >= shb, the last group of
    every batch element (rolled rows N-G..N-1: tokens N-G+shift..N-1, then the wrapped tokens
    0..shift-1) is reordered so the wrapped tokens come first (np.roll by +shift within the
    group); ``inverse`` puts them back."""
    if not enabled:
        return x
    if not 0 < shift < G:
        raise ValueError("the wrap group exists for 0 < shift < G")
    out = x.copy()
    ng = N // G
    last = slice(ng - 1, None, ng)
    out[last, :, shb:] = np.roll(x[last, :, shb:], -shift if inverse else shift, axis=1)
    return out


def _pad_rows(x: np.ndarray, N: int, Np: int) -> np.ndarray:
    """x [B, N, ...] extended with zero rows to [B, Np, ...] (Np >= N)."""
    if Np == N:
        return x
    pad = np.zeros((x.shape[0], Np - N) + x.shape[2:])
    return np.concatenate([x, pad], axis=1)


def _check_groups(N, G, partial_last_group, wrap_own_group, wrap_front_first):
    if wrap_own_group and wrap_front_first:
        raise ValueError("Variant 2 and Variant 3 are alternatives")
    if N % G != 0:
        if not partial_last_group:
            raise ValueError("the view into groups needs G to divide N")
        if wrap_own_group or wrap_front_first:
            raise ValueError("the variants are defined for G dividing N")
    return -(-N // G) * G


def s2attn_forward(q, k, v, G, scale, shift_head_begin=None, shift=None, wrap_own_group=False,
                   wrap_front_first=False, partial_last_group=False):
    """S²-Attn forward. q [B,N,Hq,d], k, v [B,N,Hkv,d] float64.

    Returns o [B,N,Hq,d] and lse [B,Hq,N], both in original token order.
    """
    B, N, Hq, d = q.shape
    Np = _check_groups(N, G, partial_last_group, wrap_own_group, wrap_front_first)
    shb, shift = _defaults(Hq, G, shift_head_begin, shift)
    splits = _wrap_splits(B, N, G, shb, shift, wrap_own_group)
    ke, ve = expand_kv(k, Hq), expand_kv(v, Hq)
    # Algorithm 1's roll: the second chunk of heads by -shift, then the view as groups.
    # (with a partial last group: pad the rolled sequence to Np rows, drop them afterwards)
    sw = lambda x: _swap_wrap_front(x, N, G, shb, shift, wrap_front_first)
    grp = lambda x: sw(_pad_rows(chunk_roll(x, -shift, shb), N, Np).reshape(B * Np // G, G, Hq, -1))
    qr, kr, vr = grp(q), grp(ke), grp(ve)
    o, lse = causal_self_attn(qr, kr, vr, scale, splits)
    o = _swap_wrap_front(o, N, G, shb, shift, wrap_front_first, inverse=True)
    lse = _swap_wrap_front(lse, N, G, shb, shift, wrap_front_first, inverse=True)
    # Algorithm 1's roll back: to [B, N, H, d], the second chunk rolled back by +shift.
    o = chunk_roll(o.reshape(B, Np, Hq, v.shape[3])[:, :N], shift, shb)
    lse = chunk_roll(lse.reshape(B, Np, Hq)[:, :N], shift, shb)
    return o, np.ascontiguousarray(lse.transpose(0, 2, 1))


def s2attn_backward(q, k, v, do, G, scale, shift_head_begin=None, shift=None,
                    wrap_own_group=False, wrap_front_first=False, partial_last_group=False):
    """Gradients of s2attn_forward's o with respect to q, k, v for upstream do [B,N,Hq,d].

    Returns dq [B,N,Hq,d], dk [B,N,Hkv,d], dv [B,N,Hkv,d] in original token order.
    """
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    Np = _check_groups(N, G, partial_last_group, wrap_own_group, wrap_front_first)
    shb, shift = _defaults(Hq, G, shift_head_begin, shift)
    splits = _wrap_splits(B, N, G, shb, shift, wrap_own_group)
    ke, ve = expand_kv(k, Hq), expand_kv(v, Hq)
    sw = lambda x: _swap_wrap_front(x, N, G, shb, shift, wrap_front_first)
    grp = lambda x: sw(_pad_rows(chunk_roll(x, -shift, shb), N, Np).reshape(B * Np // G, G, Hq, -1))
    qr, kr, vr, dor = grp(q), grp(ke), grp(ve), grp(do)
    dq, dk, dv = causal_self_attn_backward(qr, kr, vr, dor, scale, splits)
    # The derivative of a reordering is the inverse reordering, that of the padding is
    # dropping the pad rows ...
    dq, dk, dv = (_swap_wrap_front(x, N, G, shb, shift, wrap_front_first, inverse=True)
                  .reshape(B, Np, Hq, d)[:, :N] for x in (dq, dk, dv))
    # ... and that of a roll is the opposite roll ...
    dq = chunk_roll(dq, shift, shb)
    dk = chunk_roll(dk, shift, shb)
    dv = chunk_roll(dv, shift, shb)
    # ... and that of the shared K/V view is the sum over the query heads sharing it.
    rep = Hq // Hkv
    dk = dk.reshape(B, N, Hkv, rep, d).sum(axis=3)
    dv = dv.reshape(B, N, Hkv, rep, d).sum(axis=3)
    return dq, dk, dv


def rolled_token_index(N: int, G: int, shift: int) -> np.ndarray:
    """Original token of every (group, in-group row) of a shifted head, as [N/G, G].

    Obtained by applying Algorithm 1's roll to the token index itself: np.roll(arange(N), -shift).
    """
    return np.roll(np.arange(N), -shift).reshape(N // G, G)


def head_group_rows(qh, kh, vh, doh, G, scale, shift, g, q_rows, kv_rows=None):
    """The S²-Attn definition for one (batch, query head) restricted to group g.

    qh, doh [N, d] and kh, vh [N, d] are that query head's sequences (kh, vh being the
    kv head it reads) in original order; ``shift`` is the head's roll (0 when unshifted).
    ``q_rows`` are in-group rows i (rolled order) whose o, lse and dq are wanted;
    ``kv_rows`` are in-group rows j whose dk, dv contributions from this head are wanted.

    Each requested row is the definition evaluated at that row: row i attends to rows
    0..i of its group, and the gradient of kv row j gathers rows i >= j (rows i < j have
    P[i, j] = 0 under the causal mask). Rows are given back with their original tokens.
    Returns a dict with 'q_tok', 'o', 'lse', 'dq' and, if kv_rows, 'kv_tok', 'dk', 'dv'.
    """
    N = qh.shape[0]
    tok = rolled_token_index(N, G, shift)[g]
    q_g = np.roll(qh, -shift, axis=0).reshape(N // G, G, -1)[g]
    k_g = np.roll(kh, -shift, axis=0).reshape(N // G, G, -1)[g]
    v_g = np.roll(vh, -shift, axis=0).reshape(N // G, G, -1)[g]
    do_g = np.roll(doh, -shift, axis=0).reshape(N // G, G, -1)[g]

    def rows_softmax(rows):
        s = scale * (q_g[rows] @ k_g.T)
        allowed = np.arange(G)[None, :] <= np.asarray(rows)[:, None]
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        return e / l, (m + np.log(l))[:, 0]

    def rows_ds(rows, p):
        dp = do_g[rows] @ v_g.T
        return p * (dp - (p * dp).sum(axis=1, keepdims=True))

    q_rows = np.asarray(q_rows)
    p, lse = rows_softmax(q_rows)
    out = {
        "q_tok": tok[q_rows],
        "o": p @ v_g,
        "lse": lse,
        "dq": scale * (rows_ds(q_rows, p) @ k_g),
    }
    if kv_rows is not None:
        kv_rows = np.asarray(kv_rows)
        rows = np.arange(int(kv_rows.min()), G)
        p2, _ = rows_softmax(rows)
        ds2 = rows_ds(rows, p2)
        out["kv_tok"] = tok[kv_rows]
        out["dv"] = p2[:, kv_rows].T @ do_g[rows]
        out["dk"] = scale * (ds2[:, kv_rows].T @ q_g[rows])
    return out


def rope_pi(x: np.ndarray, base: float = 10000.0, pi_scale: float = 1.0,
            inverse: bool = False) -> np.ndarray:
    """Rotary position embedding with Position Interpolation, the step just before the
    attention (summary page, §3 Phase 1 step 2 "Position Embedding Modification" and §4
    "Model setup": RoPE with positions rescaled by Position Interpolation).

    The pages give no formula; this is the textbook rotary embedding in the half-split pairing
    that Llama uses: for token t (original order) and i < d/2, the pair (x[i], x[i + d/2]) is
    rotated by the angle (t * pi_scale) * base^(-2i/d). Position Interpolation multiplies the
    positions by pi_scale = (pre-trained context) / (extended context), e.g. 4096 / 8192.
    ``inverse`` rotates by the opposite angle: the transpose of the rotation, which maps the
    gradient with respect to the rotated tensor back to the input.

    x [B, N, H, d] float64; returns a new array.
    """
    B, N, H, d = x.shape
    half = d // 2
    theta = base ** (-2.0 * np.arange(half) / d)                 # [d/2]
    ang = (np.arange(N) * pi_scale)[:, None] * theta[None, :]    # [N, d/2]
    c, s = np.cos(ang)[None, :, None, :], np.sin(ang)[None, :, None, :]
    if inverse:
        s = -s
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
