"""The global attention kernel's synchronisation protocol, modelled and checked on the CPU.

`k_attn_tc` (csrc/attention_tc.cu) runs five kinds of roles in one CTA that meet only on
mbarriers and two named barriers: the Q/K producer, the V producer, the MMA thread, and two
softmax groups of four warps (one per 128-query tile).  This file restates each role's waits and
arrivals in Python, in the kernel's order, over a CTA's sequence of work items:

- the K and V rings (four stages each), the double-buffered Q tiles;
- S, P and O hand-overs per query tile (sfull / sfree / pready / pvdone / ofree);
- the MMA thread issuing an item's last PV products after the next item's first S products;
- each softmax thread reading an item's O out after the next item's first P store;
- warps whose rows lie past the row end (they keep every wait and arrival, skip the math);
- the two groups taking turns at the exponentials across items (named barriers 1 and 2):
  group 1 hands over its last tile only when the next item has two tiles, group 0 waits at an
  item's first tile only when the previous one had two tiles.

Random interleavings of the roles must all finish: no state where every unfinished role waits
(a deadlock), and no warp arriving twice on a named barrier before the barrier completes
(hardware barriers count threads, so such an arrival would pair the wrong phases).  mbarrier
waits use phase parity exactly as the kernel does.  Two planted protocol errors must be caught,
which shows the checks have teeth.  This checks the protocol as restated here, not the compiled
kernel; the source checks below tie the restatement to the constants and hand-off conditions in
the CUDA file, so a change there fails this test until the model is brought along.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(__file__), "..", "encoder_decision_model_b200", "csrc", "attention_tc.cu")


def _source():
    return open(SRC).read()


def _constants():
    src = _source()
    nk = int(re.search(r"constexpr int NK = (\d+);", src).group(1))
    nv = int(re.search(r"constexpr int NV = (\d+);", src).group(1))
    return nk, nv


def test_model_matches_the_kernel_source():
    src = _source()
    # barrier arrival counts: one arrival per softmax warp for sfree, pready and ofree
    for name in ("sfree", "pready", "ofree"):
        assert re.search(rf"mbar_init\(&{name}\[i\], 4\);", src), name
    for name in ("sfull", "pvdone", "qfull", "qfree"):
        assert re.search(rf"mbar_init\(&{name}\[i\], 1\);", src), name
    # the hand-off conditions the model restates (live and dead paths)
    assert src.count("if (j != 0 || g0_wait_first) named_bar_sync(BAR_G1_DONE, 256);") == 2
    assert src.count("else if (j != t.nt - 1 || g1_hand_last) named_bar_arrive(BAR_G1_DONE, 256);") == 2
    assert "const bool g0_wait_first = pp && prev_pp;" in src
    # the deferred last PV and the deferred readout
    assert "if (j == 0 && pend) {" in src
    assert "if (j != 0 || rd_pend) mbar_wait(&pvdone[x], (c - 1) & 1, status);" in src
    assert "if (rd_pend) readout();" in src


class _MBar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending, self.phase = 0, self.phase + 1

    def ready(self, parity):  # mbarrier.try_wait.parity: the phase of this parity has completed
        return (self.phase & 1) != parity


class _NamedBar:  # bar.sync / bar.arrive over 8 warps (256 threads)
    def __init__(self):
        self.gen, self.arrived = 0, set()

    def join(self, who):
        if who in self.arrived:
            raise AssertionError(f"warp {who} arrived twice on a named barrier")
        self.arrived.add(who)
        g = self.gen
        if len(self.arrived) == 8:
            self.gen, self.arrived = self.gen + 1, set()
        return g


def _run(items, seed, nk, nv, plant=None, p_rescale=0.25):
    rng = random.Random(seed)
    bars = {}
    for i in range(nk):
        bars[f"kfull{i}"], bars[f"kfree{i}"] = _MBar(1), _MBar(1)
    for i in range(nv):
        bars[f"vfull{i}"], bars[f"vfree{i}"] = _MBar(1), _MBar(1)
    for i in range(2):
        for n, cnt in (("qfull", 1), ("qfree", 1), ("sfull", 1), ("sfree", 4), ("pready", 4), ("pvdone", 1),
                       ("ofree", 4)):
            bars[f"{n}{i}"] = _MBar(cnt)
    named = {"G0": _NamedBar(), "G1": _NamedBar()}

    def producer():
        J = 0
        for it, t in enumerate(items):
            qbuf = it & 1
            if it >= 2:
                yield ("wait", f"qfree{qbuf}", ((it - 2) >> 1) & 1)
            yield ("arrive", f"qfull{qbuf}")
            for _ in range(t["nt"]):
                s = J % nk
                if J >= nk:
                    yield ("wait", f"kfree{s}", ((J - nk) // nk) & 1)
                yield ("arrive", f"kfull{s}")
                J += 1

    def vproducer():
        J = 0
        for t in items:
            for _ in range(t["nt"]):
                s = J % nv
                if J >= nv:
                    yield ("wait", f"vfree{s}", ((J - nv) // nv) & 1)
                yield ("arrive", f"vfull{s}")
                J += 1

    def mma():
        J, cnt, uses, pend = 0, [0, 0], [0, 0], None

        def issue_pv(Jp, nx, cx, first, us):
            s = Jp % nv
            yield ("wait", f"vfull{s}", (Jp // nv) & 1)
            for x in range(nx):
                yield ("wait", f"pready{x}", cx[x] & 1)
                if first and us[x] >= 1:
                    yield ("wait", f"ofree{x}", (us[x] - 1) & 1)
                yield ("arrive", f"pvdone{x}")
            yield ("arrive", f"vfree{s}")

        for it, t in enumerate(items):
            qbuf = it & 1
            yield ("wait", f"qfull{qbuf}", (it >> 1) & 1)
            J0, c0, u0 = J, cnt[:], uses[:]
            for j in range(t["nt"]):
                s = J % nk
                yield ("wait", f"kfull{s}", (J // nk) & 1)
                for x in range(t["nx"]):
                    c = cnt[x]
                    cnt[x] += 1
                    if c >= 1:
                        yield ("wait", f"sfree{x}", (c - 1) & 1)
                    yield ("arrive", f"sfull{x}")
                yield ("arrive", f"kfree{s}")
                if j == t["nt"] - 1:
                    yield ("arrive", f"qfree{qbuf}")
                if j == 0 and pend:
                    yield from issue_pv(*pend)
                    pend = None
                if j >= 1:
                    yield from issue_pv(J0 + j - 1, t["nx"], [c0[0] + j - 1, c0[1] + j - 1], j == 1, u0)
                J += 1
            pend = (J0 + t["nt"] - 1, t["nx"], [c0[0] + t["nt"] - 1, c0[1] + t["nt"] - 1], t["nt"] == 1, u0)
            for x in range(t["nx"]):
                uses[x] += 1
        if pend:
            yield from issue_pv(*pend)

    def softmax(x, quarter):
        who = (x, quarter)
        c, prev_pp, rd_pend = 0, False, False
        for k, t in enumerate(items):
            pp = t["nx"] == 2
            g0_wait_first = pp and prev_pp
            if plant == "group0_never_waits_first":
                g0_wait_first = False
            prev_pp = pp
            if x >= t["nx"]:
                continue
            nxt = items[k + 1] if k + 1 < len(items) else None
            g1_hand_last = pp and x == 1 and nxt is not None and nxt["nx"] == 2
            if plant == "group1_always_hands_last":
                g1_hand_last = pp and x == 1
            nt = t["nt"]
            dead = quarter * 32 >= t["rows"][x]
            if dead and rd_pend:
                yield ("wait", f"pvdone{x}", (c - 1) & 1)
                yield ("arrive", f"ofree{x}")
                rd_pend = False
            for j in range(nt):
                yield ("wait", f"sfull{x}", c & 1)
                yield ("arrive", f"sfree{x}")
                if not dead and j >= 1 and rng.random() < p_rescale:  # the running max moved: rescale O
                    yield ("wait", f"pvdone{x}", (c - 1) & 1)
                if pp:
                    if x == 0:
                        if j != 0 or g0_wait_first:
                            yield ("nsync", "G1", who)
                    else:
                        yield ("nsync", "G0", who)
                if j != 0 or (rd_pend and not dead):
                    yield ("wait", f"pvdone{x}", (c - 1) & 1)
                if pp:
                    if x == 0:
                        yield ("narrive", "G0", who)
                    elif j != nt - 1 or g1_hand_last:
                        yield ("narrive", "G1", who)
                if rd_pend and not dead:  # the previous item's O read out
                    yield ("arrive", f"ofree{x}")
                    rd_pend = False
                yield ("arrive", f"pready{x}")
                c += 1
            if dead:
                yield ("wait", f"pvdone{x}", (c - 1) & 1)
                yield ("arrive", f"ofree{x}")
            else:
                rd_pend = True
        if rd_pend:
            yield ("wait", f"pvdone{x}", (c - 1) & 1)
            yield ("arrive", f"ofree{x}")

    roles = {"producer": producer(), "v_producer": vproducer(), "mma": mma()}
    for x in range(2):
        for q in range(4):
            roles[f"softmax{x}{q}"] = softmax(x, q)
    op, done = {}, set()
    for k, g in roles.items():
        try:
            op[k] = next(g)
        except StopIteration:
            done.add(k)

    def runnable(o):
        if o[0] == "wait":
            return bars[o[1]].ready(o[2])
        if o[0] == "nsync_wait":
            return named[o[1]].gen > o[2]
        return True

    while len(done) < len(roles):
        ready = [k for k in roles if k not in done and runnable(op[k])]
        if not ready:
            stuck = ", ".join(f"{k} {op[k]}" for k in roles if k not in done)
            raise AssertionError(f"deadlock: {stuck}")
        k = rng.choice(ready)
        o = op[k]
        if o[0] == "arrive":
            bars[o[1]].arrive()
        elif o[0] == "narrive":
            named[o[1]].join(o[2])
        elif o[0] == "nsync":
            op[k] = ("nsync_wait", o[1], named[o[1]].join(o[2]))
            continue
        try:
            op[k] = next(roles[k])
        except StopIteration:
            done.add(k)
    for n, nb in named.items():  # every hand-over met its wait
        assert not nb.arrived, f"named barrier {n} ends with {len(nb.arrived)} unmatched warps"


def _items(rng, n):
    out = []
    for _ in range(n):
        nx = rng.choice([1, 2, 2, 2])
        rows = [128, rng.randint(1, 128)] if nx == 2 else [rng.randint(1, 128), 0]
        out.append({"nx": nx, "nt": rng.randint(1, 9), "rows": rows})
    return out


def test_random_interleavings_finish():
    nk, nv = _constants()
    for seed in range(400):
        rng = random.Random(7000 + seed)
        _run(_items(rng, rng.randint(0, 12)), seed, nk, nv)


def test_long_rows_and_single_tile_items():
    nk, nv = _constants()
    rng = random.Random(3)
    for seed in range(40):
        # long rows (many key steps per item), with single-tile items and dead warps between them
        items = [{"nx": 2, "nt": 64, "rows": [128, 128]}, {"nx": 1, "nt": 64, "rows": [5, 0]},
                 {"nx": 2, "nt": 64, "rows": [128, 33]}, {"nx": 2, "nt": 1, "rows": [128, 1]}]
        rng.shuffle(items)
        _run(items, seed, nk, nv)


@pytest.mark.parametrize("plant", ["group1_always_hands_last", "group0_never_waits_first"])
def test_planted_protocol_errors_are_caught(plant):
    nk, nv = _constants()
    caught = 0
    for seed in range(100):
        rng = random.Random(9000 + seed)
        try:
            _run(_items(rng, rng.randint(2, 12)), seed, nk, nv, plant=plant)
        except AssertionError:
            caught += 1
    assert caught > 0, plant
