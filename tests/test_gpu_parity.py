"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Tolerances (per row, against the float64 oracle):
  BF16 mode, and FP8 mode (E4M3 encoder QKV projections) at the same bounds:
             |delta logit| <= 3e-2, |delta p| <= 5e-3, same argmax where the
             oracle's top-2 gap exceeds 0.05; relative L2 error of the encoder
             output and of the marker states <= 3e-2.
  FP32 mode  |delta logit| <= 1e-3, |delta p| <= 1e-4, relative L2 error of
             the taps <= 1e-4.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import Row, rows_config0, rows_config1, rows_config2, write_weights
from gpu_helpers import device_run, oracle_run, compare

pytestmark = pytest.mark.gpu

OPT0 = dict(max_length=8192, head_budget=256, strict=True)
OPT1 = dict(max_length=1024, head_budget=512, strict=True)


@pytest.fixture(scope="module")
def lib_built():
    from encoder_decision_model_b200.build import build
    build()
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return jl.lib()


@pytest.fixture(scope="module")
def fp32_model(lib_built, weights_file):
    m = jl.Model(weights_file, 65536, 256, 4096, precision=jl.JD_PREC_FP32)
    yield m
    m.close()


@pytest.fixture(scope="module")
def fp8_model(lib_built, weights_file):
    m = jl.Model(weights_file, 65536, 256, 4096, precision=jl.JD_PREC_FP8)
    yield m
    m.close()


@pytest.fixture(scope="module")
def bf16_model(lib_built, weights_file):
    m = jl.Model(weights_file, 65536, 256, 4096, precision=jl.JD_PREC_BF16)
    yield m
    m.close()


def edge_rows():
    """Ragged lengths around the 64-token tile and the 129-key window."""
    rng = np.random.default_rng(77)
    ids = lambda n: rng.integers(10, 256000, size=n).astype(np.int32)
    rows = []
    for total, k, qtype in ((6, 2, 0), (63, 3, 1), (64, 2, 2), (65, 4, 0), (66, 5, 1), (127, 20, 0),
                            (128, 7, 1), (129, 2, 2), (130, 9, 0), (200, 11, 1), (257, 6, 0), (321, 2, 2)):
        small = total < 20
        olens = [0 if small else int(rng.integers(0, 4)) for _ in range(k)]
        nq = 0 if small else 3
        head = 3 + nq + k + sum(olens)
        ns = total - head - 1
        assert ns >= 0
        rows.append(Row(state=ids(ns), question=ids(nq), options=[ids(n) for n in olens], qtype=qtype))
    return rows


@pytest.mark.parametrize("cfg", ["c0", "c1", "c2", "edge"])
def test_fp32_mode_matches_oracle(fp32_model, weights_file, cfg):
    rows, opts = {"c0": (rows_config0(), OPT0), "c1": (rows_config1(), OPT1),
                  "c2": (rows_config2(12), OPT1), "edge": (edge_rows(), OPT1)}[cfg]
    hb, res = device_run(fp32_model, rows, opts, taps=True)
    ref = oracle_run(weights_file, rows, opts)
    compare(hb, res, ref, bf16=False, label=f"fp32 {cfg}")


@pytest.mark.parametrize("cfg", ["c0", "c1", "c2", "edge"])
def test_fp8_qkv_mode_matches_oracle_at_bf16_bounds(fp8_model, weights_file, cfg):
    rows, opts = {"c0": (rows_config0(), OPT0), "c1": (rows_config1(), OPT1),
                  "c2": (rows_config2(12), OPT1), "edge": (edge_rows(), OPT1)}[cfg]
    hb, res = device_run(fp8_model, rows, opts, taps=True)
    ref = oracle_run(weights_file, rows, opts)
    compare(hb, res, ref, bf16=True, label=f"fp8 {cfg}")


@pytest.mark.parametrize("cfg", ["c0", "c1", "c2", "edge"])
def test_bf16_matches_oracle(bf16_model, weights_file, cfg):
    rows, opts = {"c0": (rows_config0(), OPT0), "c1": (rows_config1(), OPT1),
                  "c2": (rows_config2(12), OPT1), "edge": (edge_rows(), OPT1)}[cfg]
    hb, res = device_run(bf16_model, rows, opts, taps=True)
    ref = oracle_run(weights_file, rows, opts)
    compare(hb, res, ref, bf16=True, label=f"bf16 {cfg}")


def test_packed_equals_rows_alone(bf16_model):
    rows = rows_config2(6)
    hb, res = device_run(bf16_model, rows, OPT1)
    for i, r in enumerate(rows):
        hb1, r1 = device_run(bf16_model, [r], OPT1)
        a, b = hb.opt_off[i], hb.opt_off[i + 1]
        np.testing.assert_allclose(res["logits"][a:b], r1["logits"], atol=1e-5)


def test_decide_host_equals_device(bf16_model):
    rows = rows_config1()
    hb, res = device_run(bf16_model, rows, OPT1)
    ho = bf16_model.jd_decide_host(rows, jl.encode_opts(**OPT1))
    np.testing.assert_array_equal(ho["logits"], res["logits"])
    np.testing.assert_array_equal(ho["choice"], res["choice"])


def _same_bucket_pair(opts):
    """Two seeded 3-question requests whose packed batches differ in length but share a graph
    bucket (tokens rounded up from T + 8 to a multiple of 128, markers from M + 1 to a multiple of 8)."""
    seen = {}
    for seed in range(101, 400):
        rows = rows_config1(seed=seed)
        hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
        key = ((hb.n_tokens + 8 + 127) // 128, hb.n_rows, (hb.n_markers + 8) // 8)
        if key in seen and seen[key][1] != hb.n_tokens:
            return seen[key][0], rows
        seen.setdefault(key, (rows, hb.n_tokens))
    raise AssertionError("no two requests share a bucket")


def test_graph_replay_equals_eager(bf16_model):
    """Graph mode against eager launches, bit for bit, on two request shapes of one bucket: the
    first call captures the bucket's graph, the second (another length, other device buffers)
    replays it; then the same two through the host entry point, and the exact-shape graph that a
    call with taps takes."""
    import torch
    ra, rb = _same_bucket_pair(OPT1)
    eager = [device_run(bf16_model, r, OPT1)[1] for r in (ra, rb)]
    eager_host = [bf16_model.jd_decide_host(r, jl.encode_opts(**OPT1)) for r in (ra, rb)]
    keys = ("logits", "probs", "choice", "score", "noul", "max_p")
    c0, r0, _ = bf16_model.jd_graph_stats()
    bf16_model.jd_set_graph_mode(True)
    try:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            for i, r in enumerate((ra, rb, ra)):
                _, res = device_run(bf16_model, r, OPT1, stream=s)
                for k in keys:
                    np.testing.assert_array_equal(res[k], eager[i % 2][k], err_msg=f"request {i % 2}: {k}")
            c1, r1, _ = bf16_model.jd_graph_stats()
            assert (c1 - c0, r1 - r0) == (1, 2), (c1 - c0, r1 - r0)
            for i, r in enumerate((ra, rb)):
                o = bf16_model.jd_decide_host(r, jl.encode_opts(**OPT1), stream=s)
                for k in keys:
                    np.testing.assert_array_equal(o[k], eager_host[i][k], err_msg=f"host request {i}: {k}")
            c2, r2, _ = bf16_model.jd_graph_stats()
            assert (c2 - c1, r2 - r1) == (0, 2), (c2 - c1, r2 - r1)
            # taps: the exact-shape graph
            tap_graph = [device_run(bf16_model, ra, OPT1, taps=True, stream=s)[1]]
            c3, _, _ = bf16_model.jd_graph_stats()
            assert c3 - c2 == 1
    finally:
        bf16_model.jd_set_graph_mode(False)
    tap_eager = device_run(bf16_model, ra, OPT1, taps=True)[1]
    for k in keys + ("encoder_out", "marker_state"):
        np.testing.assert_array_equal(tap_graph[0][k], tap_eager[k], err_msg=f"taps: {k}")
    for k in keys:
        np.testing.assert_array_equal(tap_eager[k], eager[0][k], err_msg=f"taps against no taps: {k}")


def test_capacity_and_status_errors(bf16_model):
    import torch
    rows = rows_config0()
    hb = jl.jd_serialize(rows, jl.encode_opts(**OPT0))
    dev = torch.device("cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    tok = hb.tokens.copy()
    tok[5] = 300000  # outside the vocabulary: the gather clamps it and flags the status word
    keep = [t(tok), t(hb.cu_seqlens), t(hb.mask_pos), t(hb.opt_off), t(hb.row_type)]
    b = jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)
    outs = [torch.empty(hb.n_markers, device=dev), torch.empty(hb.n_markers, device=dev),
            torch.empty(1, dtype=torch.int32, device=dev)] + [torch.empty(1, device=dev) for _ in range(3)]
    bf16_model.jd_decide(b, *outs)
    with pytest.raises(jl.JDError) as ei:
        bf16_model.jd_check_status()
    assert ei.value.code == jl.JD_ERR_DEVICE_STATUS
    big = jl.Model.device_batch(1, 10 ** 6, 3, 47, *keep)
    with pytest.raises(jl.JDError) as ei:
        bf16_model.jd_decide(big, *outs)
    assert ei.value.code == jl.JD_ERR_CAPACITY
    # a clean call afterwards clears the status word
    keep[0] = t(hb.tokens)
    b = jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)
    bf16_model.jd_decide(b, *outs)
    bf16_model.jd_check_status()


def test_scorer_and_activation_variants(lib_built, weights_file):
    rows = rows_config1()
    for scorer, act in ((jl.JD_SCORER_LINEAR, jl.JD_ACT_RELU), (jl.JD_SCORER_MLP, jl.JD_ACT_GELU)):
        m = jl.Model(weights_file, 4096, 16, 256, precision=jl.JD_PREC_BF16, scorer=scorer, head_act=act)
        hb, res = device_run(m, rows, OPT1, taps=True)
        ref = oracle_run(weights_file, rows, OPT1, scorer="linear" if scorer else "mlp",
                         head_act="gelu" if act else "relu")
        compare(hb, res, ref, bf16=True, label=f"variant scorer={scorer} act={act}")
        m.close()


def test_sharpened_scorer_argmax(lib_built, tmp_path_factory):
    """Scorer output weights x40 so that top-2 gaps exceed 0.05 and the argmax
    agreement rule is exercised on most rows."""
    p = tmp_path_factory.mktemp("w") / "sharp.jdw"
    write_weights(p, seed=0, overrides={"scorer.linear2.W": lambda a: a * 40.0})
    m = jl.Model(p, 65536, 256, 4096)
    rows = rows_config2(16)
    hb, res = device_run(m, rows, OPT1, taps=True)
    ref = oracle_run(p, rows, OPT1)
    checked = 0
    for i, r in ref.items():
        a, b = hb.opt_off[i], hb.opt_off[i + 1]
        zr = np.sort(r["logits"])[::-1]
        if zr[0] - zr[1] > 0.05:
            checked += 1
            assert res["choice"][i] == int(np.argmax(r["logits"]))
        # logits scale x40 with the weights: bound the error relative to that scale
        assert np.abs(res["logits"][a:b] - r["logits"]).max() <= 40 * 3e-2
    assert checked >= 4, checked
    m.close()
