"""Index arithmetic of the +-64 sliding-window attention kernel, checked on the CPU.

The kernel gives each CTA 64 queries [q0, q0 + 64) of one row and head and loads
the 192-key band [q0 - 64, q0 + 128); warp w (16 queries) visits LW_CHUNKS
16-key chunks starting at chunk w of the band, and tests the +-64 window only
on the outer 8-key blocks (the `edge` condition); every other block is inside
the window by construction.  This test reads the chunk count and the edge
condition from the CUDA source and checks, for every lane of the m16n8k16
fragment layout (query rows g and g + 8, key columns 2 tq + e of each 8-key
block), that (1) the skipped blocks hold only keys within 64 of the query, (2)
the warp's keys include every key within 64 of each of its queries, and (3)
they stay inside the CTA's band.
"""
import os
import re

SRC = os.path.join(os.path.dirname(__file__), "..", "encoder_decision_model_b200", "csrc", "attention.cu")
WINDOW = 64
BQ = 64


def _kernel_constants():
    src = open(SRC).read()
    chunks = int(re.search(r"constexpr int LW_CHUNKS = (\d+);", src).group(1))
    m = re.search(r"const bool edge = j < (\d+) \|\| j >= 2 \* LW_CHUNKS - (\d+);", src)
    assert m, "edge condition not found in the local attention kernel"
    return chunks, int(m.group(1)), int(m.group(2))


def test_skipped_blocks_lie_inside_the_window():
    chunks, lo, hi = _kernel_constants()
    blocks = 2 * chunks
    seen_outside_on_edges = False
    for warp in range(4):
        for lane in range(32):
            g, tq = lane >> 2, lane & 3
            q0 = 1000
            kbase = q0 - WINDOW
            qi0 = q0 + warp * 16 + g
            for qi in (qi0, qi0 + 8):
                for j in range(blocks):
                    edge = j < lo or j >= blocks - hi
                    for e in range(2):
                        kj = kbase + (warp * 2 + j) * 8 + 2 * tq + e
                        inside = abs(qi - kj) <= WINDOW
                        if not edge:
                            assert inside, (warp, lane, qi, j, e)
                        elif not inside:
                            seen_outside_on_edges = True
    # the edge blocks do need the test: some of their keys fall outside the window
    assert seen_outside_on_edges


def test_warp_keys_cover_each_query_window_and_stay_in_the_band():
    chunks, _, _ = _kernel_constants()
    q0 = 5000
    band = range(q0 - WINDOW, q0 + BQ + WINDOW)
    assert len(band) == 192
    for warp in range(4):
        keys = set(range(q0 - WINDOW + 16 * warp, q0 - WINDOW + 16 * (warp + chunks)))
        assert keys <= set(band), warp
        for r in range(16):
            qi = q0 + 16 * warp + r
            need = set(range(qi - WINDOW, qi + WINDOW + 1))
            assert need <= keys, (warp, r)


def test_interior_warps_skip_row_tests_only_when_every_key_is_in_the_row():
    """The kernel takes the copy of the mask loop without per-key row tests when the warp's
    first key kw and its last key kw + 16 * LW_CHUNKS - 1 lie in [cs, ce); brute force over
    rows of every length up to 400 and every warp position: then every key the warp reads
    is in the row, and a warp that fails the test does read a key outside it."""
    src = open(SRC).read()
    assert "if (kw >= cs && kw + 16 * LW_CHUNKS <= ce) {" in src
    chunks, _, _ = _kernel_constants()
    cs = 1000
    for L in range(1, 400):
        ce = cs + L
        for q0 in range(cs, ce, BQ):
            for warp in range(4):
                kw = q0 - WINDOW + 16 * warp
                keys = range(kw, kw + 16 * chunks)
                interior = kw >= cs and kw + 16 * chunks <= ce
                assert interior == all(cs <= k < ce for k in keys), (L, q0, warp)
