"""The moment exchange of the column-split residual + LayerNorm GEMM, modelled on the CPU.

`k_gemm_rlp` (csrc/gemm.cu) splits a tile's 384 columns over the two CTAs of a cluster.  Both
CTAs walk the same tiles in the same order; tile tc of a CTA uses TMEM accumulator and moment
buffer b = tc & 1.  Per tile:

- the MMA thread waits until the epilogue has released accumulator b (from tile tc - 2), issues
  the products and commits accf[b];
- the epilogue waits for accf[b]; its leader arms the CTA's own momf[b] with one arrival and the
  tile's expected bytes (both CTAs' moments); every epilogue thread sends its rows' (mean, M2) of
  every chunk to slot [b][chunk][row] of both CTAs as `st.async` stores, each completing its bytes
  on the receiving CTA's momf[b]; the epilogue then waits for its momf[b] phase, merges the slots,
  runs pass 2 and releases accumulator b.

An mbarrier phase completes when its pending arrival count and its transaction count are both
zero; bytes may land before the arrival that announces them (the count goes below zero for a
while).  The model delivers every CTA's stores in pieces, at random times and in random order,
and checks that (1) whenever a momf phase completes, every slot it covers holds this tile's
moments (no early completion on a later tile's bytes), (2) no store overwrites a slot its CTA
has not merged yet, and (3) every interleaving finishes.  A planted error (moment slots not
double-buffered by tile parity) must be caught.  The source checks tie the model to the kernel.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "encoder_decision_model_b200", "csrc", "gemm.cu")
NS, PIECES = 2, 3


def test_model_matches_the_kernel_source():
    src = open(SRC).read()
    i = src.index("k_gemm_rlp(")
    body = src[i:i + 20000]
    assert "mbar_init(&momf[b], 1);" in body
    assert "if (leader) mbar_arrive_expect_tx(&momf[b], NS * C::NX * 128 * 8);" in body
    assert "mbarrier::complete_tx::bytes" in body
    assert "mbar_wait_cluster(&momf[b], (tc >> 1) & 1, ep.status);" in body
    assert "if (tc >= 2 && !mbar_wait(&acce[b], ((tc >> 1) - 1) & 1, ep.status)) break;" in body
    assert re.search(r"mbar_wait\(&accf\[b\], \(tc >> 1\) & 1, ep\.status\);", body)


class _TxBar:
    """mbarrier with one expected arrival per phase and a transaction count."""

    def __init__(self):
        self.phase, self.arrivals, self.tx = 0, 1, 0

    def _maybe_complete(self):
        if self.arrivals == 0 and self.tx == 0:
            self.phase += 1
            self.arrivals = 1
            return True
        return False

    def arrive_expect(self, nbytes):
        self.tx += nbytes
        self.arrivals -= 1
        return self._maybe_complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        return self._maybe_complete()

    def ready(self, parity):
        return (self.phase & 1) != parity


def _run(n_tiles, seed, plant=None):
    rng = random.Random(seed)
    nbuf = 1 if plant == "single_moment_buffer" else 2
    momf = [[_TxBar() for _ in range(2)] for _ in range(NS)]
    accf = [[0, 0] for _ in range(NS)]  # completed phases
    acce = [[0, 0] for _ in range(NS)]
    # slot[cta][buf][sender][piece] = tile whose moments it holds; merged[cta][buf] = tiles merged
    slot = [[[[None] * PIECES for _ in range(NS)] for _ in range(nbuf)] for _ in range(NS)]
    merged = [[set() for _ in range(nbuf)] for _ in range(NS)]
    network = []  # (receiver, buf, sender, piece, tile)
    mma_tc = [0] * NS
    epi_tc = [0] * NS
    epi_step = [0] * NS  # 0: wait accf, then arm and send; 1: wait momf, then merge and release

    def on_phase_complete(r, b, tile):
        sb = b % nbuf
        for snd in range(NS):
            for p in range(PIECES):
                assert slot[r][sb][snd][p] == tile, (
                    f"CTA {r} buffer {b} completed for tile {tile} with slot {snd}/{p} holding "
                    f"{slot[r][sb][snd][p]}")

    while True:
        moves = []
        for c in range(NS):
            t = mma_tc[c]
            if t < n_tiles and (t < 2 or acce[c][t & 1] >= (t >> 1)):
                moves.append(("mma", c))
            t = epi_tc[c]
            if t < n_tiles:
                b = t & 1
                if epi_step[c] == 0 and accf[c][b] > (t >> 1):
                    moves.append(("send", c))
                elif epi_step[c] == 1 and momf[c][b].ready((t >> 1) & 1):
                    moves.append(("merge", c))
        if network:
            moves.append(("deliver", None))
        if not moves:
            break
        kind, c = rng.choice(moves)
        if kind == "mma":
            t = mma_tc[c]
            accf[c][t & 1] += 1
            mma_tc[c] += 1
        elif kind == "send":
            t = epi_tc[c]
            b = t & 1
            if momf[c][b].arrive_expect(NS * PIECES):  # the leader arms its own barrier
                on_phase_complete(c, b, 2 * (momf[c][b].phase - 1) + b)
            for r in range(NS):
                for p in range(PIECES):
                    network.append((r, b, c, p, t))
            epi_step[c] = 1
        elif kind == "deliver":
            r, b, snd, p, t = network.pop(rng.randrange(len(network)))
            sb = b % nbuf
            prev = slot[r][sb][snd][p]
            assert prev is None or prev in merged[r][sb], (
                f"tile {t} from CTA {snd} overwrote CTA {r}'s unmerged moments of tile {prev}")
            slot[r][sb][snd][p] = t
            if momf[r][b].complete_tx(1):
                # phase k of buffer b belongs to the receiver's tile 2 k + b
                on_phase_complete(r, b, 2 * (momf[r][b].phase - 1) + b)
        else:  # merge, pass 2, release the accumulator
            t = epi_tc[c]
            b = t & 1
            sb = b % nbuf
            for snd in range(NS):
                for p in range(PIECES):
                    assert slot[c][sb][snd][p] == t, f"CTA {c} merged tile {t} with stale moments"
            merged[c][sb].add(t)
            acce[c][b] += 1
            epi_tc[c] += 1
            epi_step[c] = 0
    assert epi_tc == [n_tiles] * NS and mma_tc == [n_tiles] * NS, (epi_tc, mma_tc)


def test_random_speeds_and_delivery_orders():
    for seed in range(3000):
        _run(random.Random(seed).randint(1, 9), seed)


def test_planted_single_moment_buffer_is_caught():
    caught = 0
    for seed in range(300):
        try:
            _run(random.Random(seed).randint(3, 9), seed, plant="single_moment_buffer")
        except AssertionError:
            caught += 1
    assert caught > 0
