"""The host FP8 E4M3 encoder that quantizes the QKV weights of the FP8 mode
(csrc/e4m3.h), compiled with g++ and compared with an encoding written here
from the format's definition: every one of the 256 codes decodes to a value;
a float encodes to the code of the nearest value (ties to the even code),
saturating at 448."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _decode(code):
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 7
    if e == 15 and m == 7:
        return np.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8.0) * 2.0 ** (e - 7)


def _reference(x):
    """Nearest finite code (ties: even mantissa), saturating; +-0 keep their sign."""
    vals = np.array([_decode(c) for c in range(256)])
    out = []
    for v in x.astype(np.float64):
        if np.isnan(v):
            out.append(0x7F)
            continue
        sign = 0x80 if np.signbit(v) else 0
        a = min(abs(v), 448.0)
        cand = [c for c in range(0x7F) if np.isfinite(vals[c])]   # non-negative codes 0x00..0x7e
        d = np.array([abs(vals[c] - a) for c in cand])
        best = np.flatnonzero(d == d.min())
        c = cand[best[0]] if len(best) == 1 else [cand[b] for b in best if cand[b] % 2 == 0][0]
        out.append(sign | c)
    return np.array(out)


@pytest.fixture(scope="module")
def encoder(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not found")
    exe = tmp_path_factory.mktemp("e4m3") / "e4m3_check"
    subprocess.run([gxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "encoder_decision_model_b200", "csrc"),
                    os.path.join(ROOT, "tests", "e4m3_check.cpp"), "-o", str(exe)], check=True)

    def run(x):
        x = np.asarray(x, np.float32)
        inp = "\n".join(f"{u:08x}" for u in x.view(np.uint32)) + "\n"
        r = subprocess.run([str(exe)], input=inp, capture_output=True, text=True, check=True)
        return np.array([int(t, 16) for t in r.stdout.split()])
    return run


def test_every_code_round_trips(encoder):
    vals = np.array([_decode(c) for c in range(256)])
    ok = np.isfinite(vals)
    got = encoder(vals[ok])
    want = np.arange(256)[ok]
    want[want == 0x80] = 0x80  # -0 keeps its sign
    np.testing.assert_array_equal(got, want)


def test_rounding_ties_and_saturation(encoder):
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 1, 2000), rng.normal(0, 50, 500), rng.uniform(-2e-3, 2e-3, 500),
                        [448.0, 449.0, 464.0, 1e6, -1e6, 0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -10, 2.0 ** -9 * 7.5,
                         1.0625, 1.1875, 240.0, 232.0]]).astype(np.float32)
    np.testing.assert_array_equal(encoder(x), _reference(x))
