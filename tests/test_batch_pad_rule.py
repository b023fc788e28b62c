"""The bucket padding of a batch for CUDA-graph replay (csrc/batch_pad.h), checked on the CPU.

A batch of T tokens, B rows and M markers replays the graph of its bucket: Tb tokens, B + 1 rows
and Mb markers, the added row (the pad row) holding tokens T .. Tb - 1 and markers M .. Mb - 1.
The header's host functions are compiled with g++ into a small harness that prints the padded
arrays of random batches; this test checks what the forward pass needs of them:

- Tb is a multiple of 128 with at least 8 pad tokens, Mb a multiple of 8 with 1 to 8 pad
  markers (every row, the pad row too, has a marker for the per-row softmax);
- the real rows' tokens, offsets, markers and types are unchanged;
- the row and marker offsets stay non-decreasing and end at Tb and Mb;
- every pad marker sits on a token of the pad row, in order, and the pad row has type 0;
- two batches with the same bucket share (Tb, Bb, Mb), so one graph serves both.
"""
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "encoder_decision_model_b200", "csrc")
CUDA_INC = "/usr/local/cuda/include"

HARNESS = r"""
#include <cstdio>
#include <vector>
#include "batch_pad.h"
int main() {
    int T, B, M;
    while (std::scanf("%d %d %d", &T, &B, &M) == 3) {
        std::vector<int> tok(T), cu(B + 1), mask(M), opt(B + 1), type(B);
        for (auto &v : tok) std::scanf("%d", &v);
        for (auto &v : cu) std::scanf("%d", &v);
        for (auto &v : mask) std::scanf("%d", &v);
        for (auto &v : opt) std::scanf("%d", &v);
        for (auto &v : type) std::scanf("%d", &v);
        const jd::PadShape s = jd::pad_shape(T, B, M);
        std::printf("%d %d %d\n", s.Tb, s.Bb, s.Mb);
        for (int i = 0; i < s.Tb; ++i) std::printf("%d ", jd::pad_token_at(s, tok.data(), i));
        std::printf("\n");
        for (int i = 0; i <= s.Bb; ++i) std::printf("%d ", jd::pad_cu_at(s, cu.data(), i));
        std::printf("\n");
        for (int i = 0; i < s.Mb; ++i) std::printf("%d ", jd::pad_mask_at(s, mask.data(), i));
        std::printf("\n");
        for (int i = 0; i <= s.Bb; ++i) std::printf("%d ", jd::pad_opt_at(s, opt.data(), i));
        std::printf("\n");
        for (int i = 0; i < s.Bb; ++i) std::printf("%d ", jd::pad_type_at(s, type.data(), i));
        std::printf("\n");
    }
    return 0;
}
"""


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None or not os.path.isdir(CUDA_INC):
        pytest.skip("g++ or the CUDA headers are not available")
    d = tmp_path_factory.mktemp("pad")
    src = d / "pad.cpp"
    src.write_text(HARNESS)
    exe = d / "pad"
    subprocess.run([gxx, "-std=c++17", "-O1", f"-I{CSRC}", f"-I{CUDA_INC}", str(src), "-o", str(exe)], check=True,
                   capture_output=True, text=True)
    return str(exe)


def _batch(rng):
    B = rng.randint(1, 12)
    lens = [rng.randint(6, 300) for _ in range(B)]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    opt, mask = [0], []
    for r in range(B):
        k = rng.randint(2, min(20, lens[r] - 2))
        pos = sorted(rng.sample(range(cu[r] + 1, cu[r + 1]), k))
        mask += pos
        opt.append(opt[-1] + k)
    T, M = cu[-1], len(mask)
    tok = [rng.randint(1, 255999) for _ in range(T)]
    typ = [rng.randint(0, 2) for _ in range(B)]
    return T, B, M, tok, cu, mask, opt, typ


def _pad(exe, batches):
    inp = []
    for T, B, M, tok, cu, mask, opt, typ in batches:
        inp.append(f"{T} {B} {M}")
        for arr in (tok, cu, mask, opt, typ):
            inp.append(" ".join(map(str, arr)) if arr else "")
    out = subprocess.run([exe], input="\n".join(inp) + "\n", capture_output=True, text=True, check=True).stdout
    lines = out.strip("\n").split("\n")
    res = []
    for i in range(len(batches)):
        Tb, Bb, Mb = map(int, lines[6 * i].split())
        arrs = [list(map(int, lines[6 * i + k].split())) for k in range(1, 6)]
        res.append(((Tb, Bb, Mb), *arrs))
    return res


def test_padded_batches_are_valid_and_keep_the_real_rows(harness):
    rng = random.Random(17)
    batches = [_batch(rng) for _ in range(300)]
    for (T, B, M, tok, cu, mask, opt, typ), ((Tb, Bb, Mb), ptok, pcu, pmask, popt, ptyp) in zip(
            batches, _pad(harness, batches)):
        assert Tb % 128 == 0 and Tb - T >= 8 and Tb - T < 8 + 128
        assert Mb % 8 == 0 and 1 <= Mb - M <= 8
        assert Bb == B + 1
        assert len(ptok) == Tb and len(pcu) == Bb + 1 and len(pmask) == Mb and len(popt) == Bb + 1
        assert len(ptyp) == Bb
        # the real rows are unchanged
        assert ptok[:T] == tok and pcu[:B + 1] == cu and pmask[:M] == mask and popt[:B + 1] == opt
        assert ptyp[:B] == typ
        # offsets
        assert all(a <= b for a, b in zip(pcu, pcu[1:])) and pcu[-1] == Tb and pcu[B] == T
        assert all(a <= b for a, b in zip(popt, popt[1:])) and popt[-1] == Mb and popt[B] == M
        # the pad row: id 0 tokens, type 0, its markers on its own first tokens, in order
        assert all(v == 0 for v in ptok[T:]) and ptyp[B] == 0
        assert pmask[M:] == list(range(T, T + (Mb - M)))
        assert all(T <= p < Tb for p in pmask[M:])


def test_one_bucket_serves_nearby_shapes(harness):
    rng = random.Random(5)
    batches = [_batch(rng) for _ in range(200)]
    for (T, B, M, *_), (shape, *_) in zip(batches, _pad(harness, batches)):
        # the documented rule, restated: at least 8 pad tokens rounded up to 128, at least one
        # pad marker rounded up to 8, one pad row
        assert shape == ((T + 8 + 127) // 128 * 128, B + 1, (M + 8) // 8 * 8)
    # a batch and the same batch with one more token in its last row share the bucket unless the
    # extra token crosses a multiple of 128
    T, B, M, tok, cu, mask, opt, typ = batches[0]
    longer = (T + 1, B, M, tok + [7], cu[:-1] + [cu[-1] + 1], mask, opt, typ)
    (s0, *_), (s1, *_) = _pad(harness, [batches[0], longer])
    assert (s0 == s1) == ((T + 8) % 128 != 0)
