"""CPU-side checks of the C ABI and of the host/index logic (no kernel is launched).

* libs2attn.so loads and exports every function include/s2attn.h declares;
* argument validation rejects bad calls before any CUDA call (fake device addresses);
* the remap and tile-order functions the kernels use (s2_tiles.cuh), compiled here with g++,
  agree with the oracle's literal roll (LongLoRA summary page, §3.4 Algorithm 1 key line 1)
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
    assert lib.s2attn_abi_version() == 2
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
    (dict(N=200), 1), (dict(G=63, N=63 * 4), 1), (dict(scale=0.0), 1),
    (dict(scale=float("nan")), 1), (dict(scale=float("inf")), 1), (dict(scale=-1.0), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(G=24, N=240), 2), (dict(G=8, N=64), 2),
    (dict(N=1 << 30, G=1 << 29), 2),
])
def test_fwd_rejects(lib, kw, status):
    assert fwd_call(lib, **kw) == status


@pytest.mark.parametrize("shb,shift,kw,status", [
    (-1, 32, {}, 1), (5, 32, {}, 1), (2, 4, {}, 2), (2, 36, {}, 2),
    # G=24: G/2 = 12 is not a multiple of 8, but a roll of 8 (or none) is fine -> reaches
    # CUDA set-up, which is not available here; we only check it is not rejected as bad shape
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
    assert lib.s2attn_bwd_dkdv(A, A, A, A, A, A, 1, 4, 4, 256, 64, 64, ctypes.c_float(0.1), 2,
                               36, ws, need, None) == 2


# --------------------------------------------------------------------------------------
# Index logic of the kernels, compiled for the host.
# --------------------------------------------------------------------------------------
SHIM = r"""
#include "s2_tiles.cuh"
extern "C" {
void rolled_runs(int r0, int shift, int N, int* o) {
  s2::TileRuns t = s2::rolled_tile_runs(r0, shift, N); o[0]=t.valid; o[1]=t.first; o[2]=t.start; }
void original_runs(int t0, int shift, int N, int* o) {
  s2::TileRuns t = s2::original_tile_runs(t0, shift, N); o[0]=t.valid; o[1]=t.first; o[2]=t.start; }
int qtiles(int t0, int sh, int N, int G, int W, int* o) {
  s2::QTileRanges q = s2::kv_tile_qtiles(t0, sh, N, G, W);
  int n = q.count(); for (int i = 0; i < n; ++i) o[i] = q.at(i); return n; }
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
void kvspan(int qt, int sh, int N, int G, int W, int* o) {
  s2::KvSpan s = s2::qtile_kv_span(qt, sh, N, G, W); o[0] = s.first; o[1] = s.count; }
long long dsslots(int N, int G, int shifted, int shift, int W, int qt) {
  s2::DsSlots d = s2::ds_slots(N, G, shifted, shift, W);
  return qt < 0 ? d.per_head : d.base(qt); }
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
    return ctypes.CDLL(str(so))


NOWRAP = 0x7FFFFFFF   # no wrap split (the default variant)


def call4(fn, *args):
    out = (ctypes.c_int * 4)()
    fn(*args, out)
    return list(out)


CASES = [(256, 64, 32), (8192, 2048, 1024), (320, 64, 32), (384, 192, 96), (200, 200, 0),
         (96, 32, 16), (1024, 1024, 512), (640, 128, 64), (2048, 512, 256), (448, 64, 8),
         (96, 96, 88), (768, 256, 640)]


@pytest.mark.parametrize("N,G,shift", CASES)
def test_rolled_runs_match_literal_roll(shim, N, G, shift):
    tok = orc.rolled_token_index(N, G, shift).reshape(-1)   # rolled row -> original token
    for r0 in range(0, N, 128):
        valid, first, start = call4(shim.rolled_runs, r0, shift, N)[:3]
        assert valid == min(128, N - r0)
        got = [start + i for i in range(first)] + [i - first for i in range(first, valid)]
        assert got == list(tok[r0:r0 + valid])
        assert first % 8 == 0 and valid % 8 == 0 and start % 8 == 0


@pytest.mark.parametrize("N,G,shift", CASES)
def test_original_runs_invert_the_roll(shim, N, G, shift):
    tok = orc.rolled_token_index(N, G, shift).reshape(-1)
    rolled_of = np.empty(N, dtype=np.int64)
    rolled_of[tok] = np.arange(N)
    for t0 in range(0, N, 128):
        valid, first, start = call4(shim.original_runs, t0, shift, N)[:3]
        got = [start + i for i in range(first)] + [i - first for i in range(first, valid)]
        assert got == list(rolled_of[t0:t0 + valid])


@pytest.mark.parametrize("N,G,shift", CASES)
def test_kv_tile_query_tiles_exact(shim, N, G, shift):
    """Brute force: q tile Qt is visited for kv tile t0 iff some rolled query row in Qt attends
    some kv row of the tile (same rolled group, query not before key)."""
    tok = orc.rolled_token_index(N, G, shift).reshape(-1)
    rolled_of = np.empty(N, dtype=np.int64)
    rolled_of[tok] = np.arange(N)
    out = (ctypes.c_int * 4096)()
    for t0 in range(0, N, 128):
        n = shim.qtiles(t0, shift, N, G, NOWRAP, out)
        got = list(out[:n])
        assert len(set(got)) == len(got)
        want = set()
        for t in range(t0, min(t0 + 128, N)):
            rk = rolled_of[t]
            ge = (rk // G + 1) * G
            want.update(range(rk // 128, (ge - 1) // 128 + 1))
        assert set(got) == want


@pytest.mark.parametrize("B,Hq,N,G", [(1, 4, 256, 64), (2, 3, 8192, 2048), (1, 2, 384, 192),
                                      (3, 2, 320, 64), (1, 1, 1024, 1024)])
def test_query_tile_order_is_a_permutation(shim, B, Hq, N, G):
    nt = (N + 127) // 128
    seen = set()
    for bid in range(B * Hq * nt):
        seen.add(tuple(call4(shim.qcoords, bid, B, Hq, N, G)[:3]))
    assert seen == {(b, h, q) for b in range(B) for h in range(Hq) for q in range(nt)}
    if G % 128 == 0 and G > 128:
        # the first wave holds the tiles with the most key tiles (last tile of each group)
        b, h, qt = call4(shim.qcoords, 0, B, Hq, N, G)[:3]
        assert qt % (G // 128) == G // 128 - 1


@pytest.mark.parametrize("B,Hq,Hkv,N,G,shb,sh", [(1, 4, 4, 256, 64, 2, 32),
                                                  (2, 8, 2, 8192, 2048, 4, 1024),
                                                  (1, 8, 1, 1024, 256, 4, 128),
                                                  (1, 4, 2, 384, 192, 2, 96),
                                                  (1, 64, 8, 32768, 8192, 32, 4096)])
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


@pytest.mark.parametrize("N,G,shift", CASES + [(102400, 25600, 12800), (32768, 8192, 4096)])
def test_qtile_kv_span_exact(shim, N, G, shift):
    """Brute force: the original kv tiles a rolled query tile reads are exactly the tiles
    holding some kv row that one of its rows attends (same rolled group, key not after query),
    listed once each from `first` on (indices modulo the tile count)."""
    nt = (N + 127) // 128
    for sh in {0, shift}:
        for qt in range(nt) if N <= 8192 else list(range(0, nt, 37)) + [nt - 1]:
            first, count = call4(shim.kvspan, qt, sh, N, G, NOWRAP)[:2]
            got = [(first + i) % nt for i in range(count)]
            assert len(set(got)) == count
            r0, last = qt * 128, min(qt * 128 + 127, N - 1)
            gb = (r0 // G) * G
            want = {((r + sh) % N) // 128 for r in range(gb, last + 1)}
            assert set(got) == want


@pytest.mark.parametrize("N,G,shift", CASES)
def test_ds_slots_match_the_dkdv_pairs(shim, N, G, shift):
    """Every (query tile, kv tile) pair the dQ pass reads is one the dK/dV kernel visits, and
    the slots of one head are distinct and inside per_head."""
    nt = (N + 127) // 128
    shim.dsslots.restype = ctypes.c_longlong
    per_head = shim.dsslots(N, G, 1, shift, NOWRAP, -1)
    out = (ctypes.c_int * 4096)()
    for sh in {0, shift}:
        visited = set()
        for t in range(nt):
            n = shim.qtiles(t * 128, sh, N, G, NOWRAP, out)
            visited.update((qt, t) for qt in out[:n])
        slots = set()
        for qt in range(nt):
            first, count = call4(shim.kvspan, qt, sh, N, G, NOWRAP)[:2]
            base = shim.dsslots(N, G, 1, shift, NOWRAP, qt)
            for i in range(count):
                assert (qt, (first + i) % nt) in visited
                slots.add(base + i)
            assert base + count <= per_head
        assert len(slots) == sum(call4(shim.kvspan, qt, sh, N, G, NOWRAP)[1] for qt in range(nt))
    if G % 128 == 0 and shift % 128 == 0:
        gt = G // 128
        assert per_head == (N // G) * gt * (gt + 1) // 2


V2_CASES = [(256, 64, 32), (8192, 2048, 1024), (320, 64, 32), (384, 192, 96), (96, 32, 16),
            (640, 128, 64), (2048, 512, 256), (448, 64, 8), (96, 96, 88), (1024, 256, 128),
            (512, 128, 40)]


def _v2_group(r, N, G, W):
    """Rolled rows of the causal group holding rolled row r when the wrapped tokens (rolled
    rows [W, N), W = N - shift) form their own group (Table 8, Variant 2)."""
    if r >= W:
        return W, N
    return (r // G) * G, min((r // G + 1) * G, W)


@pytest.mark.parametrize("N,G,shift", V2_CASES)
def test_variant2_tile_sets_exact(shim, N, G, shift):
    """Brute force with the wrap split: the query tiles each kv tile visits, the kv tiles each
    query tile reads, and that the two agree in both directions (every dS tile the dK/dV kernel
    hands off lands inside the reading tile's span, and every span entry is written)."""
    W = N - shift
    nt = (N + 127) // 128
    tok = orc.rolled_token_index(N, G, shift).reshape(-1)
    rolled_of = np.empty(N, dtype=np.int64)
    rolled_of[tok] = np.arange(N)
    out = (ctypes.c_int * 4096)()
    visited = set()
    for t in range(nt):
        n = shim.qtiles(t * 128, shift, N, G, W, out)
        got = set(out[:n])
        assert len(got) == n
        want = set()
        for tk in range(t * 128, min(t * 128 + 128, N)):
            rk = rolled_of[tk]
            want.update(range(rk // 128, (_v2_group(rk, N, G, W)[1] - 1) // 128 + 1))
        assert got == want
        visited.update((qt, t) for qt in got)
    shim.dsslots.restype = ctypes.c_longlong
    per_head = shim.dsslots(N, G, 1, shift, W, -1)
    read, slots = set(), set()
    for qt in range(nt):
        first, count = call4(shim.kvspan, qt, shift, N, G, W)[:2]
        got = [(first + i) % nt for i in range(count)]
        assert len(set(got)) == count
        r0, last = qt * 128, min(qt * 128 + 127, N - 1)
        gb = _v2_group(r0, N, G, W)[0]
        assert set(got) == {((r + shift) % N) // 128 for r in range(gb, last + 1)}
        read.update((qt, t) for t in got)
        base = shim.dsslots(N, G, 1, shift, W, qt)
        assert base + count <= per_head
        slots.update(base + i for i in range(count))
    assert read == visited
    assert len(slots) == len(read)
    # the default variant's slot layout holds at least as many tiles per head
    assert per_head >= shim.dsslots(N, G, 1, shift, NOWRAP, -1) or G % 128 or shift % 128


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
    assert lib.s2attn_fwd_general(*ok_args, 2, None, None) == 1
    no_roll = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 4, 32]
    assert lib.s2attn_fwd_general(*no_roll, 1, None, None) == 1
    zero_shift = [A] * 5 + [2, 4, 4, 256, 64, 64, f, 2, 0]
    assert lib.s2attn_fwd_general(*zero_shift, 1, None, None) == 1
