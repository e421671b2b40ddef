"""The work decomposition of the tensor-core SCA kernels, checked on the CPU.

The forward kernel (sca_tc.cu) hands out work units of two 128-row query
tiles through decode_unit; the backward kernels (sca_bwd_tc.cu) give each CTA
one 128-row tile through bwd_tile.  Both functions are compiled here from the
kernel sources as plain host C++ (g++) and enumerated over many shapes,
including chunk sizes that are odd multiples of 128, odd tile counts and
segments with a prepended previous chunk.  The checks are the sliding chunk
window of the Gecko digest (method step details, step 3; paperlayer.ai
summary, section 3.2), restated here: every query tile is covered exactly
once, and its key range runs from the start of the previous chunk (the
sequence start for chunk 1) to the diagonal tile; for the key-side backward,
every key tile is covered once with the query tiles that see it."""
import os
import re
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "long_context_sequence_sca_b200",
                    "csrc")
TILE = 128

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")


def _block(src: str, start: str) -> str:
    """The text from `start` to the brace that closes its first block."""
    i = src.index(start)
    j = src.index("{", i)
    depth = 0
    for k in range(j, len(src)):
        if src[k] == "{":
            depth += 1
        elif src[k] == "}":
            depth -= 1
            if depth == 0:
                end = k + 1
                if src[end:end + 1] == ";":
                    end += 1
                return src[i:end]
    raise ValueError(f"unbalanced block after {start!r}")


def _host_source() -> str:
    fwd = open(os.path.join(CSRC, "sca_tc.cu")).read()
    bwd = open(os.path.join(CSRC, "sca_bwd_tc.cu")).read()
    kbn = re.search(r"constexpr int kBN = (\d+);", fwd).group(1)
    krows = re.search(r"constexpr int kRows = (\d+);", bwd)
    krows = krows.group(1) if krows else str(TILE)
    parts = [
        "#include <cstdio>\n#include <cstdint>\n#include <cstdlib>\n",
        "#define __device__\n#define __forceinline__ inline\n",
        f"constexpr int kBN = {kbn};\nconstexpr int kRows = {krows};\n",
        _block(fwd, "struct Unit {"),
        _block(fwd, "__device__ __forceinline__ Unit decode_unit("),
        _block(bwd, "struct BwdTile {"),
        _block(bwd, "__device__ __forceinline__ BwdTile bwd_tile("),
        r'''
int main(int argc, char** argv) {
  const int BH = atoi(argv[1]), T = atoi(argv[2]), c = atoi(argv[3]), koff = atoi(argv[4]);
  const int n_units = BH * ((T + 255) / 256);
  for (int u = 0; u < n_units; ++u) {
    Unit U = decode_unit(u, BH, T, c, koff);
    printf("U %lld %d %d %d %d %d %d\n", (long long)U.bh, U.q0, U.nt, U.beg[0], U.end[0], U.beg[1], U.end[1]);
  }
  const int grid = BH * (T / kRows);
  for (int b = 0; b < grid; ++b) {
    BwdTile k = bwd_tile(b, T, c, false), q = bwd_tile(b, T, c, true);
    printf("K %lld %d %d %d\nQ %lld %d %d %d\n", (long long)k.bh, k.row, k.beg, k.end, (long long)q.bh, q.row,
           q.beg, q.end);
  }
  return 0;
}
''',
    ]
    return "\n".join(parts)


def _compile(text: str, name: str) -> str:
    d = os.path.join(os.path.dirname(CSRC), "..", "_build", "schedule_check")
    os.makedirs(d, exist_ok=True)
    src, out = os.path.join(d, name + ".cpp"), os.path.join(d, name)
    with open(src, "w") as f:
        f.write(text)
    subprocess.run(["g++", "-O1", "-std=c++17", "-o", out, src], check=True, capture_output=True)
    return out


@pytest.fixture(scope="module")
def exe():
    return _compile(_host_source(), "sched")


def _run(exe, BH, T, c, koff):
    lines = subprocess.run([exe, str(BH), str(T), str(c), str(koff)], check=True, capture_output=True,
                           text=True).stdout.split("\n")
    units = [tuple(map(int, ln.split()[1:])) for ln in lines if ln.startswith("U ")]
    ktiles = [tuple(map(int, ln.split()[1:])) for ln in lines if ln.startswith("K ")]
    qtiles = [tuple(map(int, ln.split()[1:])) for ln in lines if ln.startswith("Q ")]
    return units, ktiles, qtiles


def _key_range(r0, c, koff):
    """Key tiles [beg, end) that 128-row query tile r0 reads: from the start
    of the previous chunk (negative rows = the prepended chunk of a continued
    segment; the sequence start for chunk 1 of a fresh one) to the diagonal."""
    ch = r0 // c
    lo = (ch - 1) * c if (ch >= 1 or koff > 0) else 0
    return lo // TILE, r0 // TILE + 1


SHAPES = [
    # BH, T, c, koff
    (1, 128, 128, 0), (3, 384, 128, 0), (2, 1024, 256, 0), (2, 1280, 256, 0), (1, 1536, 384, 0),
    (5, 2304, 384, 0), (4, 4096, 512, 0), (3, 3072, 1024, 0), (2, 8192, 4096, 0), (7, 640, 128, 0),
    (2, 1024, 256, 256), (3, 1536, 384, 384), (1, 768, 128, 128), (2, 8192, 4096, 4096),
]


@pytest.mark.parametrize("BH,T,c,koff", SHAPES)
def test_forward_units_cover_each_query_tile_once_with_its_window(exe, BH, T, c, koff):
    units, _, _ = _run(exe, BH, T, c, koff)
    assert len(units) == BH * ((T + 255) // 256)
    seen = {}
    for bh, q0, nt, b0, e0, b1, e1 in units:
        assert 0 <= bh < BH and q0 % 256 == 0 and nt in (1, 2)
        assert nt == (2 if q0 + TILE < T else 1)
        for i, (b, e) in enumerate(((b0, e0), (b1, e1))[:nt]):
            r0 = q0 + TILE * i
            assert r0 < T
            key = (bh, r0 // TILE)
            assert key not in seen, f"query tile {key} twice"
            seen[key] = (b, e)
            assert (b, e) == _key_range(r0, c, koff), (key, (b, e))
    assert len(seen) == BH * (T // TILE)


@pytest.mark.parametrize("BH,T,c,koff", [s for s in SHAPES if s[3] == 0])
def test_backward_tiles_cover_each_tile_once(exe, BH, T, c, koff):
    _, ktiles, qtiles = _run(exe, BH, T, c, koff)
    n = T // TILE
    tpc = c // TILE
    assert sorted((bh, row) for bh, row, _, _ in ktiles) == [(b, r) for b in range(BH) for r in range(n)]
    assert sorted((bh, row) for bh, row, _, _ in qtiles) == [(b, r) for b in range(BH) for r in range(n)]
    for bh, row, beg, end in qtiles:
        assert (beg, end) == _key_range(row * TILE, c, 0)
    for bh, row, beg, end in ktiles:
        # query tiles that see key tile `row`: causal from the diagonal, up to
        # the end of the chunk after the key's chunk
        want = [qt for qt in range(n) if row <= qt and qt // tpc <= row // tpc + 1]
        assert (beg, end) == (want[0], want[-1] + 1), (bh, row, beg, end)


@pytest.mark.parametrize("c", [128, 256, 384, 1024])
def test_window_rule_matches_the_oracle_mask(c):
    """The tile-level window used above equals the union, over the rows of
    the tile, of the oracle's per-token window [window_lo(t), t]; so a key
    tile is read iff some row of the query tile sees a key in it."""
    from oracle.gecko_oracle import window_lo
    T = 6 * c
    for r0 in range(0, T, TILE):
        tiles = set()
        for t in range(r0, r0 + TILE):
            tiles.update(range(window_lo(t, c) // TILE, t // TILE + 1))
        assert (min(tiles), max(tiles) + 1) == _key_range(r0, c, 0)
        assert tiles == set(range(min(tiles), max(tiles) + 1))


@pytest.mark.parametrize("old,new", [
    ("U.beg[i] = lo / kBN;", "U.beg[i] = lo / kBN + 1;"),          # window starts one tile late
    ("const int o = npc - 1 - u % npc;", "const int o = u % npc / 2;"),  # units collide
    ("? (ch + 2) * tpc : n_tiles", "? (ch + 1) * tpc : n_tiles"),   # next chunk's queries dropped
])
def test_a_planted_schedule_mistake_is_caught(old, new):
    """The same checks on a copy of the functions with one plausible slip
    (compiled on the CPU only) must fail."""
    text = _host_source()
    assert text.count(old) == 1
    exe = _compile(text.replace(old, new), "sched_mutant")
    caught = False
    for BH, T, c, koff in SHAPES:
        try:
            test_forward_units_cover_each_query_tile_once_with_its_window(exe, BH, T, c, koff)
            if koff == 0:
                test_backward_tiles_cover_each_tile_once(exe, BH, T, c, koff)
        except AssertionError:
            caught = True
            break
    assert caught
