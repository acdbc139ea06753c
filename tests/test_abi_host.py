"""CPU-side checks of the C ABI and of the host/index logic (no kernel is launched).

* libs2attn.so loads and exports every function include/s2attn.h declares;
* argument validation rejects bad calls before any CUDA call (fake device addresses);
* the remap and tile-order functions the kernels use (s2_tiles.cuh), compiled here with g++,
  agree with the oracle's literal roll (LongLoRA summary page, §3.4 Algorithm 1, the roll before the attention)
  and with a brute-force enumeration of which query rows see which key rows.
"""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import s2attn_oracle as orc
import shifted_sparse_attention_fwd_b200 as s2
from shifted_sparse_attention_fwd_b200 import build as s2build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s2attn.h")
CSRC = os.path.join(ROOT, "shifted_sparse_attention_fwd_b200", "csrc")


@pytest.fixture(scope="module")
def lib():
    s2build.build()
    return s2.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(s2attn_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(s2.SIGNATURES), set(names) ^ set(s2.SIGNATURES)
    out = subprocess.run(["nm", "-D", "--defined-only", s2.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported
    # Nothing else leaks out of the library (hidden visibility by default).
    assert {e for e in exported if e.startswith("s2attn_")} == set(names)


def test_version_and_status_strings(lib):
    assert lib.s2attn_abi_version() == 5
    for st in range(5):
        assert s2.status_string(st)
    assert s2.status_string(99) == "unknown status"
    # D and LSE2 (each rounded up to 256 bytes), then 256 bytes of work counters
    assert lib.s2attn_bwd_workspace_size(1, 32, 8192) == 2 * 32 * 8192 * 4 + 256
    assert lib.s2attn_bwd_workspace_size(1, 1, 8) == 3 * 256
    assert lib.s2attn_bwd_workspace_size(0, 1, 8) == 0


A = 0x10000  # fake, 16-byte aligned device addresses: validation must reject before use


def fwd_call(lib, **kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, Hq=4, Hkv=4, N=256, d=64, G=64, scale=0.125)
    a.update(kw)
    return lib.s2attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                          a["N"], a["d"], a["G"], a["scale"], None)


def fwd_ex_call(lib, shb, shift, **kw):
    a = dict(B=1, Hq=4, Hkv=4, N=256, d=64, G=64, scale=0.125)
    a.update(kw)
    return lib.s2attn_fwd_ex(A, A, A, A, A, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["G"],
                             a["scale"], shb, shift, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(k=A + 8), 1), (dict(o=A + 2), 1),
    (dict(B=0), 1), (dict(N=-8), 1), (dict(Hq=3, Hkv=3), 1), (dict(Hkv=3), 1),
    (dict(N=200), 1), (dict(scale=0.0), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1), (dict(scale=-1.0), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(N=1 << 30, G=1 << 29), 2),
])
def test_fwd_rejects(lib, kw, status):
    assert fwd_call(lib, **kw) == status


@pytest.mark.parametrize("shb,shift,kw,status", [
    (-1, 32, {}, 1), (5, 32, {}, 1), (5, 4, {}, 1),
])
def test_fwd_ex_rejects(lib, shb, shift, kw, status):
    assert fwd_ex_call(lib, shb, shift, **kw) == status


def test_bwd_rejects(lib):
    ws = 0x100000
    need = lib.s2attn_bwd_workspace_size(1, 4, 256)
    args = [A] * 9 + [1, 4, 4, 256, 64, 64, ctypes.c_float(0.125)]
    assert lib.s2attn_bwd(*args, None, need, None) == 1                  # null workspace
    assert lib.s2attn_bwd(*args, ws + 16, need, None) == 1               # misaligned
    assert lib.s2attn_bwd(*args, ws, need - 4, None) == 1                # too small
    bad = [A] * 8 + [None] + [1, 4, 4, 256, 64, 64, ctypes.c_float(0.125)]
    assert lib.s2attn_bwd(*bad, ws, need, None) == 1                     # null dv
    odd = [A] * 9 + [1, 3, 3, 256, 64, 64, ctypes.c_float(0.125)]
    assert lib.s2attn_bwd(*odd, ws, need, None) == 1                     # odd Hq
    d96 = [A] * 9 + [1, 4, 4, 256, 96, 64, ctypes.c_float(0.125)]
    assert lib.s2attn_bwd(*d96, ws, need, None) == 2
    assert lib.s2attn_bwd_preprocess(A, A, A, 1, 4, 256, 64, ws, 8, None) == 1
    assert lib.s2attn_bwd_preprocess(A, A, A, 1, 4, 256, 80, ws, need, None) == 2
    assert lib.s2attn_bwd_dq(A, A, A, A, None, 1, 4, 4, 256, 64, 64, ctypes.c_float(0.1), 2,
                             32, ws, need, None) == 1
    assert lib.s2attn_bwd_dkdv(A, A, A, A, A, A, 1, 4, 4, 256, 96, 64, ctypes.c_float(0.1), 2,
                               36, ws, need, None) == 2


@pytest.mark.parametrize("B,Hq,Hkv,N,d,G,shb,shift,flags", [
    (1, 32, 32, 8192, 128, 1365, 16, 682, 4),   # the page's 1/6 group (Table 7), rolled by 682
    (1, 4, 4, 300, 64, 75, 2, 37, 0),           # odd G, odd roll
    (1, 4, 2, 1000, 64, 333, 2, 166, 4),        # odd G, shorter last group
    (1, 4, 4, 693, 64, 231, 2, 115, 1),         # odd G, Variant 2
    (1, 4, 4, 512, 128, 128, 2, 37, 2),         # a roll of 37, Variant 3
    (2, 2, 2, 129, 64, 43, 1, 21, 0),           # N, G, roll all odd
    (1, 2, 2, 250, 64, 24, 1, 12, 4),           # G/2 not a multiple of 8
])
def test_any_group_and_roll_accepted(lib, B, Hq, Hkv, N, d, G, shb, shift, flags):
    """G and the roll need not be multiples of 8 (nor G even): validation accepts them (the
    workspace query runs the same checks without touching a device)."""
    assert lib.s2attn_bwd_workspace_size_general(B, Hq, Hkv, N, d, G, shb, shift, flags, 0) > 0


# --------------------------------------------------------------------------------------
# Index logic of the kernels, compiled for the host.
# --------------------------------------------------------------------------------------
SHIM = r"""
#include "s2_tiles.cuh"
#include "s2_fwd_sched.h"
extern "C" {
int fwdlists(int B, int Hq, int N, int G, int shb, int wrap, int grid, int* start, int* unit) {
  std::vector<int> s, u;
  if (!s2::fwd_unit_lists(B, Hq, N, G, shb, wrap, grid, s, u)) return -1;
  std::copy(s.begin(), s.end(), start);
  std::copy(u.begin(), u.end(), unit);
  return static_cast<int>(u.size()); }
static void put_runs(const s2::Runs& t, int* o) {
  o[0] = t.n; o[1] = t.valid;
  for (int k = 0; k < t.n; ++k) { o[2 + 2 * k] = t.len[k]; o[3 + 2 * k] = t.src[k]; } }
void rolled_runs(int r0, int shift, int N, int G, int front, int* o) {
  put_runs(s2::rolled_runs(s2::head_remap(N, G, shift, front), r0), o); }
unsigned straddled(int r0, int shift, int N, int G, int front) {
  return s2::straddled_atoms(s2::rolled_runs(s2::head_remap(N, G, shift, front), r0)); }
unsigned past_end(int r0, int shift, int N, int G, int front) {
  return s2::past_end_atoms(s2::rolled_runs(s2::head_remap(N, G, shift, front), r0)); }
void token_runs(int t0, int shift, int N, int G, int front, int* o) {
  put_runs(s2::token_runs(s2::head_remap(N, G, shift, front), t0), o); }
int qtiles(int t0, int sh, int N, int G, int W, int front, int* o) {
  s2::QTileRanges q = s2::kv_tile_qtiles(s2::head_remap(N, G, sh, front), t0, W);
  int n = q.count(); for (int i = 0; i < n; ++i) o[i] = q.at(i); return n; }
int kvspan(int qt, int sh, int N, int G, int W, int front, int* o) {
  s2::KvSpan s = s2::qtile_kv_span(s2::head_remap(N, G, sh, front), qt, W);
  int n = s.count(); for (int i = 0; i < n; ++i) o[i] = s.at(i);
  for (int i = 0; i < n; ++i) if (s.index_of(o[i]) != i) return -1;
  return n; }
long long dsslots(int N, int G, int shifted, int shift, int W, int front, int qt) {
  s2::DsSlots d = s2::ds_slots(N, G, shifted, shift, W, front);
  return qt < 0 ? d.per_head : d.base(qt); }
void qcoords(int bid, int B, int Hq, int N, int G, int* o) {
  s2::query_tile_coords(bid, B, Hq, N, G, o[0], o[1], o[2]); }
void paircoords(int bid, int B, int Hq, int N, int G, int* o) {
  s2::query_pair_coords(bid, B, Hq, N, G, o[0], o[1], o[2]); o[3] = s2::query_pairs_per_head(N); }
void kvcoords(int bid, int B, int Hq, int Hkv, int N, int G, int shb, int sh, int* o) {
  s2::kv_tile_coords(bid, B, Hq, Hkv, N, G, shb, sh, o[0], o[1], o[2]); }
void qcoords_chunked(int bid, int B, int Hq, int N, int G, int chunk, int* o) {
  s2::query_tile_coords_chunked(bid, B, Hq, N, G, chunk, o[0], o[1], o[2]); }
void paircoords_chunked(int bid, int B, int Hq, int N, int G, int chunk, int* o) {
  s2::query_pair_coords_chunked(bid, B, Hq, N, G, chunk, o[0], o[1], o[2]); }
void kvcoords_chunked(int bid, int B, int Hq, int Hkv, int N, int G, int shb, int sh, int chunk,
                      int* o) {
  s2::kv_tile_coords_chunked(bid, B, Hq, Hkv, N, G, shb, sh, chunk, o[0], o[1], o[2]); }
}
"""


@pytest.fixture(scope="module")
def shim(tmp_path_factory):
    d = tmp_path_factory.mktemp("shim")
    src = d / "shim.cpp"
    src.write_text(SHIM)
    so = d / "shim.so"
    subprocess.run(["g++", "-O1", "-shared", "-fPIC", "-std=c++17", "-I", CSRC, str(src), "-o",
                    str(so)], check=True)
    lib_ = ctypes.CDLL(str(so))
    lib_.dsslots.restype = ctypes.c_longlong
    return lib_


NOWRAP = 0x7FFFFFFF   # no wrap split (the default variant)


def call4(fn, *args):
    out = (ctypes.c_int * 4)()
    fn(*args, out)
    return list(out)


def runs_of(fn, *args):
    """[(len, src), ...] and the valid row count of a Runs result."""
    out = (ctypes.c_int * 8)()
    fn(*args, out)
    n, valid = out[0], out[1]
    return [(out[2 + 2 * k], out[3 + 2 * k]) for k in range(n)], valid


def listed(fn, *args):
    out = (ctypes.c_int * 4096)()
    n = fn(*args, out)
    assert n >= 0, "index_of disagrees with at"
    return list(out[:n])


CASES = [(256, 64, 32), (8192, 2048, 1024), (320, 64, 32), (384, 192, 96), (200, 200, 0),
         (96, 32, 16), (1024, 1024, 512), (640, 128, 64), (2048, 512, 256), (448, 64, 8),
         (96, 96, 88), (768, 256, 640),
         # G or the roll not a multiple of 8 (runs that start or end inside an 8-row atom)
         (300, 75, 37), (129, 43, 21), (512, 128, 37), (250, 50, 25), (693, 231, 115)]
# (N, G, shift) with 0 < shift < G: the cases where Variants 2 and 3 exist
SPLIT_CASES = [(256, 64, 32), (8192, 2048, 1024), (320, 64, 32), (384, 192, 96), (96, 32, 16),
               (640, 128, 64), (2048, 512, 256), (448, 64, 8), (96, 96, 88), (1024, 256, 128),
               (512, 128, 40), (1024, 1024, 512), (256, 256, 200), (136, 136, 8),
               (300, 75, 37), (693, 231, 115), (512, 128, 37), (129, 129, 5), (384, 192, 101)]
# (N, G, shift) with G not dividing N: the last rolled group is shorter
PARTIAL_CASES = [(320, 128, 64), (200, 64, 32), (136, 64, 32), (264, 256, 128), (72, 128, 64),
                 (8832, 2048, 1024), (1000, 96, 48), (384, 256, 0),
                 # the page's 1/6 group of 8192 tokens (Table 7) and other odd shapes
                 (8192, 1365, 682), (1000, 333, 166), (8191, 1365, 682), (77, 100, 50)]
VARIANT_CASES = ([(n, g, s, "default") for n, g, s in CASES + PARTIAL_CASES] +
                 [(n, g, s, v) for n, g, s in SPLIT_CASES for v in ("v2", "v3")])


def rolled_tokens(N, G, shift, variant):
    """Original token of every rolled row of a shifted head, from the oracle's own steps:
    Algorithm 1's roll, then (Variant 3) the oracle's reordering of the last group."""
    if variant != "v3":
        return np.roll(np.arange(N), -shift)
    tok = orc.rolled_token_index(N, G, shift)
    tok = orc._swap_wrap_front(tok[:, :, None], N, G, 0, shift, True)[:, :, 0]
    return tok.reshape(-1)


def groups(N, G, shift, variant):
    """group id of every rolled row (Variant 2 splits the last group at N - shift)."""
    gid = np.arange(N) // G
    if variant == "v2":
        gid = np.where(np.arange(N) >= N - shift, N // G, gid)
    return gid


def variant_args(N, shift, variant):
    return (N - shift if variant == "v2" else NOWRAP), (1 if variant == "v3" else 0)


@pytest.mark.parametrize("N,G,shift,variant", VARIANT_CASES)
def test_rolled_runs_match_the_oracle(shim, N, G, shift, variant):
    """Runs of a rolled tile give exactly the oracle's token of every row; runs of an
    original tile give the inverse; the 8-row atoms that straddle two runs (loaded with plain
    loads, not TMA boxes) are exactly the ones marked."""
    tok = rolled_tokens(N, G, shift, variant)
    rolled_of = np.empty(N, dtype=np.int64)
    rolled_of[tok] = np.arange(N)
    front = 1 if variant == "v3" else 0
    for x0 in range(0, N, 128):
        for fn, ref in ((shim.rolled_runs, tok), (shim.token_runs, rolled_of)):
            runs, valid = runs_of(fn, x0, shift, N, G, front)
            assert valid == min(128, N - x0)
            got = [src + i for ln, src in runs for i in range(ln)]
            assert got == list(ref[x0:x0 + valid])
            assert 1 <= len(runs) <= 3
        # atoms (8 rows) that hold rows of two runs are exactly those marked for plain loads
        runs, valid = runs_of(shim.rolled_runs, x0, shift, N, G, front)
        run_of_row = [k for k, (ln, _) in enumerate(runs) for _ in range(ln)]
        want = 0
        for a in range(16):
            if len({run_of_row[r] for r in range(8 * a, min(8 * a + 8, valid))}) > 1:
                want |= 1 << a
        assert shim.straddled(x0, shift, N, G, front) == want
        # tile stores (rotated queries): an atom sent as one 8-row box must have its 8 rows in
        # the sequence on 8 consecutive tokens; every atom reaching past the end, and every
        # atom whose tokens are not consecutive, is left to row-by-row stores
        past = shim.past_end(x0, shift, N, G, front)
        skip = shim.straddled(x0, shift, N, G, front) | past
        for a in range(16):
            rows = list(range(x0 + 8 * a, x0 + 8 * a + 8))
            boxable = rows[-1] < N and all(tok[r] == tok[rows[0]] + i for i, r in enumerate(rows))
            assert bool((past >> a) & 1) == (rows[-1] >= N), (x0, a)
            if not (skip >> a) & 1:
                assert boxable, (x0, a)


@pytest.mark.parametrize("N,G,shift,variant", VARIANT_CASES)
def test_tile_sets_exact(shim, N, G, shift, variant):
    """Brute force over rows: the query tiles each kv tile visits (increasing, each once) and
    the kv tiles each query tile reads (each once) are exactly the tiles holding a (query,
    key) pair of the same group with the key not after the query in rolled order."""
    nt = (N + 127) // 128
    W, front = variant_args(N, shift, variant)
    tok = rolled_tokens(N, G, shift, variant)
    rolled_of = np.empty(N, dtype=np.int64)
    rolled_of[tok] = np.arange(N)
    gid = groups(N, G, shift, variant)
    gend = np.empty(N, dtype=np.int64)      # one past the last rolled row of each row's group
    for g in np.unique(gid):
        rows = np.nonzero(gid == g)[0]
        gend[rows] = rows.max() + 1
    pairs = set()
    for t in range(nt):
        got = listed(shim.qtiles, t * 128, shift, N, G, W, front)
        assert got == sorted(set(got))
        want = set()
        for tk in range(t * 128, min(t * 128 + 128, N)):
            rk = rolled_of[tk]
            want.update(range(rk // 128, (gend[rk] - 1) // 128 + 1))
        assert set(got) == want
        pairs.update((qt, t) for qt in got)
    for qt in range(nt):
        got = listed(shim.kvspan, qt, shift, N, G, W, front)
        assert len(set(got)) == len(got)
        r0, last = qt * 128, min(qt * 128 + 127, N - 1)
        gb = np.nonzero(gid == gid[r0])[0].min()
        assert set(got) == {tok[r] // 128 for r in range(gb, last + 1)}
        for t in got:
            assert (qt, t) in pairs


@pytest.mark.parametrize("N,G,shift,variant", VARIANT_CASES)
def test_ds_slots_match_the_dkdv_pairs(shim, N, G, shift, variant):
    """Every (query tile, kv tile) pair the dQ pass reads is one the dK/dV kernel visits and
    vice versa, for both head kinds, and the slots of one head are distinct and inside
    per_head."""
    nt = (N + 127) // 128
    W, front = variant_args(N, shift, variant)
    per_head = shim.dsslots(N, G, 1, shift, W, front, -1)
    for sh, w, fr in {(0, NOWRAP, 0), (shift, W if shift else NOWRAP, front if shift else 0)}:
        visited = set()
        for t in range(nt):
            visited.update((qt, t) for qt in listed(shim.qtiles, t * 128, sh, N, G, w, fr))
        read, slots = set(), set()
        for qt in range(nt):
            span = listed(shim.kvspan, qt, sh, N, G, w, fr)
            base = shim.dsslots(N, G, 1, shift, W, front, qt)
            assert base + len(span) <= per_head
            read.update((qt, t) for t in span)
            slots.update(base + i for i in range(len(span)))
        assert read == visited
        assert len(slots) == len(read)
    if N % G == 0 and G % 128 == 0 and shift % 128 == 0 and variant == "default":
        gt = G // 128
        assert per_head == (N // G) * gt * (gt + 1) // 2


@pytest.mark.parametrize("N,G,shift", [(102400, 25600, 12800), (32768, 8192, 4096)])
def test_qtile_kv_span_large(shim, N, G, shift):
    """The long-sequence workloads, sampled: spans are the kv tiles of the group start up to
    the query tile, under the roll."""
    nt = (N + 127) // 128
    for sh in (0, shift):
        for qt in list(range(0, nt, 37)) + [nt - 1]:
            got = listed(shim.kvspan, qt, sh, N, G, NOWRAP, 0)
            r0, last = qt * 128, min(qt * 128 + 127, N - 1)
            gb = (r0 // G) * G
            assert len(set(got)) == len(got)
            assert set(got) == {((r + sh) % N) // 128 for r in range(gb, last + 1)}


@pytest.mark.parametrize("B,Hq,N,G", [(1, 4, 256, 64), (2, 3, 8192, 2048), (1, 2, 384, 192),
                                      (3, 2, 320, 64), (1, 1, 1024, 1024), (1, 4, 320, 128),
                                      (2, 2, 8832, 2048)])
def test_query_tile_order_is_a_permutation(shim, B, Hq, N, G):
    nt = (N + 127) // 128
    seen = set()
    for bid in range(B * Hq * nt):
        seen.add(tuple(call4(shim.qcoords, bid, B, Hq, N, G)[:3]))
    assert seen == {(b, h, q) for b in range(B) for h in range(Hq) for q in range(nt)}
    if N % G == 0 and G % 128 == 0 and G > 128:
        # the first wave holds the tiles with the most key tiles (last tile of each group)
        b, h, qt = call4(shim.qcoords, 0, B, Hq, N, G)[:3]
        assert qt % (G // 128) == G // 128 - 1


@pytest.mark.parametrize("B,Hq,Hkv,N,G,shb,sh", [(1, 4, 4, 256, 64, 2, 32),
                                                  (2, 8, 2, 8192, 2048, 4, 1024),
                                                  (1, 8, 1, 1024, 256, 4, 128),
                                                  (1, 4, 2, 384, 192, 2, 96),
                                                  (1, 64, 8, 32768, 8192, 32, 4096),
                                                  (1, 4, 4, 320, 128, 2, 64),
                                                  (2, 4, 2, 8832, 2048, 2, 1024)])
def test_kv_tile_order_is_a_permutation(shim, B, Hq, Hkv, N, G, shb, sh):
    nt = (N + 127) // 128
    seen = set()
    for bid in range(B * Hkv * nt):
        b, kvh, t0 = call4(shim.kvcoords, bid, B, Hq, Hkv, N, G, shb, sh)[:3]
        assert t0 % 128 == 0
        seen.add((b, kvh, t0 // 128))
    assert seen == {(b, k, t) for b in range(B) for k in range(Hkv) for t in range(nt)}


@pytest.mark.parametrize("B,Hq,N,G", [(1, 4, 256, 64), (2, 3, 8192, 2048), (1, 2, 384, 192),
                                      (3, 2, 320, 64), (1, 1, 1024, 1024), (1, 2, 640, 128),
                                      (1, 2, 16, 16)])
def test_query_pair_order_is_a_permutation(shim, B, Hq, N, G):
    nt = (N + 127) // 128
    npair = call4(shim.paircoords, 0, B, Hq, N, G)[3]
    assert npair == (nt + 1) // 2
    seen = set()
    for bid in range(B * Hq * npair):
        seen.add(tuple(call4(shim.paircoords, bid, B, Hq, N, G)[:3]))
    assert seen == {(b, h, p) for b in range(B) for h in range(Hq) for p in range(npair)}
    if G % 256 == 0 and G > 256:
        b, h, p = call4(shim.paircoords, 0, B, Hq, N, G)[:3]
        assert p % (G // 256) == G // 256 - 1


def test_fwd_rope_q_rejects(lib):
    f = ctypes.c_float(0.125)
    ok = [A] * 6 + [1, 4, 4, 256, 64, 64, f, 2, 32, 0]
    assert lib.s2attn_fwd_rope_q(*([A] * 5), None, *ok[6:], ctypes.c_float(10000.0),
                                 ctypes.c_float(1.0), None) == 1                  # no q_rot
    assert lib.s2attn_fwd_rope_q(*([A] * 5), A + 8, *ok[6:], ctypes.c_float(10000.0),
                                 ctypes.c_float(1.0), None) == 1                  # misaligned
    assert lib.s2attn_fwd_rope_q(*ok, ctypes.c_float(1.0), ctypes.c_float(1.0), None) == 1  # base
    assert lib.s2attn_fwd_rope_q(*ok, ctypes.c_float(10000.0), ctypes.c_float(0.0), None) == 1
    bad_d = [A] * 6 + [1, 4, 4, 256, 96, 64, f, 2, 32, 0]
    assert lib.s2attn_fwd_rope_q(*bad_d, ctypes.c_float(10000.0), ctypes.c_float(1.0), None) == 2


def test_rope_rejects(lib):
    """Argument checks of s2attn_rope_pi, before any launch."""
    f = ctypes.c_float
    ok = [A, A, 1, 64, 4, 128]
    assert lib.s2attn_rope_pi(None, A, 1, 64, 4, 128, f(1e4), f(0.5), 0, None, None) == 1
    assert lib.s2attn_rope_pi(A + 8, A, 1, 64, 4, 128, f(1e4), f(0.5), 0, None, None) == 1
    assert lib.s2attn_rope_pi(*ok, f(1.0), f(0.5), 0, None, None) == 1      # base <= 1
    assert lib.s2attn_rope_pi(*ok, f(1e4), f(0.0), 0, None, None) == 1      # pi_scale <= 0
    assert lib.s2attn_rope_pi(*ok, f(1e4), f(0.5), 2, None, None) == 1      # inverse not 0/1
    assert lib.s2attn_rope_pi(A, A, 1, 64, 4, 96, f(1e4), f(0.5), 0, None, None) == 2
    bad = (ctypes.c_longlong * 4)(*[4 * 128 * 64, 4 * 128 - 8] * 2)      # token stride < H*d
    assert lib.s2attn_rope_pi(*ok, f(1e4), f(0.5), 0, bad, None) == 1


def test_workspace_size_ex(lib):
    base = lib.s2attn_bwd_workspace_size(1, 32, 8192)
    full = lib.s2attn_bwd_workspace_size_ex(1, 32, 32, 8192, 128, 2048, 16, 1024, 0)
    assert full == base + 32 * (4 * 16 * 17 // 2) * 32768           # 544 tiles per head
    one = lib.s2attn_bwd_workspace_size_ex(1, 32, 32, 8192, 128, 2048, 16, 1024, 1)
    assert one == base + 544 * 32768                                  # at least one kv head
    capped = lib.s2attn_bwd_workspace_size_ex(1, 32, 32, 8192, 128, 2048, 16, 1024, base + 5 * 544 * 32768 + 7)
    assert capped == base + 5 * 544 * 32768
    gqa = lib.s2attn_bwd_workspace_size_ex(1, 64, 8, 32768, 128, 8192, 32, 4096, 0)
    assert gqa == lib.s2attn_bwd_workspace_size(1, 64, 32768) + 64 * (4 * 64 * 65 // 2) * 32768
    assert lib.s2attn_bwd_workspace_size_ex(1, 3, 3, 256, 64, 64, 1, 32, 0) > 0
    assert lib.s2attn_bwd_workspace_size_ex(1, 4, 4, 256, 96, 64, 2, 32, 0) == 0   # d = 96
    assert lib.s2attn_bwd_workspace_size_ex(1, 4, 3, 256, 64, 64, 2, 32, 0) == 0   # Hq % Hkv


def test_ds_entries_reject(lib):
    ws = 0x100000
    small = lib.s2attn_bwd_workspace_size(1, 4, 256)
    full = lib.s2attn_bwd_workspace_size_ex(1, 4, 4, 256, 64, 64, 2, 32, 0)
    f = ctypes.c_float(0.125)
    assert lib.s2attn_bwd_dkdv_ds(A, A, A, A, A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, ws, small,
                                  None) == 1                          # no room for dS
    assert lib.s2attn_bwd_dq_ds(A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, ws, full - 16,
                                None) == 1
    assert lib.s2attn_bwd_dq_ds(A, None, 1, 4, 4, 256, 64, 64, f, 2, 32, ws, full, None) == 1
    assert lib.s2attn_bwd_dq_ds(A, A, 1, 4, 4, 256, 96, 64, f, 2, 32, ws, full, None) == 2
    # the _general forms: flags and strides are validated before the workspace size
    full2 = lib.s2attn_bwd_workspace_size_general(1, 4, 4, 256, 64, 64, 2, 32, 1, 0)
    assert full2 > 0
    assert lib.s2attn_bwd_dkdv_ds_general(A, A, A, A, A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, 8,
                                          None, ws, full2, None) == 1   # unknown flag bit
    assert lib.s2attn_bwd_dkdv_ds_general(A, A, A, A, A, A, 1, 4, 4, 256, 64, 64, f, 4, 32, 1,
                                          None, ws, full2, None) == 1   # Variant 2, no rolled head
    assert lib.s2attn_bwd_dkdv_ds_general(A, A, A, A, A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, 1,
                                          None, ws, small, None) == 1   # no room for dS
    assert lib.s2attn_bwd_dq_ds_general(A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, 2, None, ws,
                                        full2 - 16, None) == 1
    bad = (ctypes.c_longlong * 16)(*([4 * 64 * 3, 4 * 64 - 8] * 8))  # token stride below H*d
    assert lib.s2attn_bwd_dq_ds_general(A, A, 1, 4, 4, 256, 64, 64, f, 2, 32, 0, bad, ws, full2,
                                        None) == 1


@pytest.mark.parametrize("B,Hq,N,G,chunk", [(1, 32, 8192, 2048, 10), (2, 3, 8192, 2048, 4),
                                            (1, 4, 256, 64, 10), (1, 2, 384, 192, 3),
                                            (3, 2, 1024, 256, 5), (1, 1, 1024, 1024, 7)])
def test_chunked_query_tile_order_is_a_permutation(shim, B, Hq, N, G, chunk):
    """The L2-grouped order visits every (b, h, tile) once; within a chunk, tiles of equal
    position in their group are adjacent and the heaviest (last in group) come first."""
    nt = (N + 127) // 128
    order = [tuple(call4(shim.qcoords_chunked, bid, B, Hq, N, G, chunk)[:3])
             for bid in range(B * Hq * nt)]
    assert set(order) == {(b, h, q) for b in range(B) for h in range(Hq) for q in range(nt)}
    if G % 128 == 0:
        tpg = G // 128
        first = order[:min(chunk, B * Hq * (N // G))]
        assert all(q % tpg == tpg - 1 for _, _, q in first)


@pytest.mark.parametrize("B,Hq,N,G,chunk", [(1, 32, 8192, 2048, 10), (2, 3, 8192, 2048, 4),
                                            (1, 4, 256, 64, 10), (1, 2, 640, 128, 3),
                                            (3, 2, 1024, 256, 5), (1, 1, 1024, 1024, 7)])
def test_chunked_pair_order_is_a_permutation(shim, B, Hq, N, G, chunk):
    nt = (N + 127) // 128
    npair = (nt + 1) // 2
    order = [tuple(call4(shim.paircoords_chunked, bid, B, Hq, N, G, chunk)[:3])
             for bid in range(B * Hq * npair)]
    assert set(order) == {(b, h, q) for b in range(B) for h in range(Hq) for q in range(npair)}


def fwd_lists(shim, B, Hq, N, G, shb, grid):
    npair = ((N + 127) // 128 + 1) // 2
    start = (ctypes.c_int * (grid + 1))()
    unit = (ctypes.c_int * (B * Hq * npair))()
    n = shim.fwdlists(B, Hq, N, G, shb, NOWRAP, grid, start, unit)
    return n, list(start), list(unit)


def pair_cost(shim, u, B, Hq, N, G):
    """The schedule's cost model restated: 3 per unit plus, for each of the pair's query tiles,
    the key tiles it visits (its own and the earlier ones of its group; no wrap split)."""
    _, _, pair = call4(shim.paircoords_chunked, u, B, Hq, N, G, 10)[:3]
    nqt = (N + 127) // 128
    c = 3
    for qt in (2 * pair, 2 * pair + 1):
        if qt < nqt:
            c += qt - (qt * 128 // G) * G // 128 + 1
    return c


@pytest.mark.parametrize("B,Hq,N,G,shb,grid", [(1, 32, 8192, 2048, 16, 148),
                                               (4, 32, 8192, 2048, 16, 148),
                                               (1, 32, 8192, 1365, 16, 148),
                                               (1, 4, 2048, 512, 2, 17),
                                               (2, 3, 1000, 333, 1, 5),
                                               (1, 8, 4096, 4096, 8, 64)])
def test_fwd_schedule_lists(shim, B, Hq, N, G, shb, grid):
    """The forward's per-CTA unit lists: every unit exactly once, each CTA's list ascending, and
    the greedy bound of list scheduling — each unit went to the least-loaded CTA, so no CTA ends
    more than one unit's cost above the mean."""
    n, start, unit = fwd_lists(shim, B, Hq, N, G, shb, grid)
    npair = ((N + 127) // 128 + 1) // 2
    assert n == B * Hq * npair
    assert start[0] == 0 and start[-1] == n and all(a <= b for a, b in zip(start, start[1:]))
    assert sorted(unit) == list(range(n))
    cost = [pair_cost(shim, u, B, Hq, N, G) for u in range(n)]
    loads = []
    for c in range(grid):
        mine = unit[start[c]:start[c + 1]]
        assert mine == sorted(mine)
        loads.append(sum(cost[u] for u in mine))
    mean = sum(cost) / grid
    assert max(loads) <= mean + max(cost)
    if (B, Hq, N, G, grid) == (1, 32, 8192, 2048, 148):
        assert max(loads) <= 1.04 * mean      # the busiest CTA about 3 % above the mean


def test_fwd_schedule_round_robin_when_units_do_not_outnumber_ctas(shim):
    assert fwd_lists(shim, 1, 2, 512, 128, 1, 148)[0] == -1    # 4 units, 148 CTAs


@pytest.mark.parametrize("B,Hq,Hkv,N,G,shb,sh,chunk", [(1, 32, 32, 8192, 2048, 16, 1024, 10),
                                                        (2, 8, 2, 8192, 2048, 4, 1024, 3),
                                                        (1, 64, 8, 32768, 8192, 32, 4096, 10),
                                                        (1, 4, 4, 256, 64, 2, 32, 10),
                                                        (1, 4, 2, 384, 192, 2, 96, 2)])
def test_chunked_kv_tile_order_is_a_permutation(shim, B, Hq, Hkv, N, G, shb, sh, chunk):
    nt = (N + 127) // 128
    order = []
    for bid in range(B * Hkv * nt):
        b, kvh, t0 = call4(shim.kvcoords_chunked, bid, B, Hq, Hkv, N, G, shb, sh, chunk)[:3]
        assert t0 % 128 == 0
        order.append((b, kvh, t0 // 128))
    assert set(order) == {(b, k, t) for b in range(B) for k in range(Hkv) for t in range(nt)}


def test_general_entries_reject(lib):
    """Stride validation happens on the host, before anything is launched."""
    f = ctypes.c_float(0.125)
    LL = ctypes.c_longlong
    good = [256 * 4 * 64 * 3, 4 * 64 * 3] * 4          # packed qkv-like strides, B = 2
    ok_args = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 2, 32]
    bad_cases = [
        [256 * 4 * 64 * 3, 4 * 64 - 8] + good[2:],      # token stride below H*d
        [256 * 4 * 64 * 3, 4 * 64 * 3 + 4] + good[2:],  # not a multiple of 8 elements
        [4 * 64 * 3, 4 * 64 * 3] + good[2:],            # batches overlap (B = 2)
    ]
    for st in bad_cases:
        arr = (LL * 8)(*st)
        assert lib.s2attn_fwd_general(*ok_args, 0, arr, None) == 1
    ws = 0x100000
    need = lib.s2attn_bwd_workspace_size(2, 4, 256)
    arr = (LL * 16)(*([4 * 64 * 3, 4 * 64 - 8] * 8))
    assert lib.s2attn_bwd_general(*([A] * 9), 2, 4, 4, 256, 64, 64, f, 2, 32, 0, arr, ws, need,
                                  None) == 1
    # option flags: unknown bits, and Variant 2 without a rolled head or with shift 0
    assert lib.s2attn_fwd_general(*ok_args, 8, None, None) == 1      # unknown bit
    assert lib.s2attn_fwd_general(*ok_args, 3, None, None) == 1      # Variants 2 and 3 together
    no_roll = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 4, 32]
    assert lib.s2attn_fwd_general(*no_roll, 1, None, None) == 1
    zero_shift = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 2, 0]
    assert lib.s2attn_fwd_general(*zero_shift, 1, None, None) == 1
    assert lib.s2attn_fwd_general(*no_roll, 2, None, None) == 1      # Variant 3, same rules
    assert lib.s2attn_fwd_general(*zero_shift, 2, None, None) == 1
    big_shift = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 2, 64]             # shift = G
    assert lib.s2attn_fwd_general(*big_shift, 2, None, None) == 1
    # G not dividing N: only with the partial-last-group flag, never with a variant
    ragged = [A] * 5 + [2, 4, 4, 320, 64, 128, f, 2, 64]
    assert lib.s2attn_fwd_general(*ragged, 0, None, None) == 1
    assert lib.s2attn_fwd_general(*ragged, 4 | 1, None, None) == 1
    assert lib.s2attn_fwd_general(*ragged, 4 | 2, None, None) == 1
