"""GPU parity at full workload sizes, on sampled outputs the oracle computes one
by one (tolerances as in test_gpu_parity.py).

  * throughput: 1024 packed rows, the batch bench.py times, in its launch
    configuration (capacity = the batch); sampled rows against the oracle;
  * long context: 16 rows x 8192 tokens; rows 0 and 9 against oracle values
    stored by tests/golden/make_long_context_golden.py;
  * router: 512 requests over 72 labels through jd_route_host (4 + 1 calls
    per request).
"""
import os

import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from oracle import EncodeOptions, readouts, serialize_row, survivors
from workloads import Row, requests_config4, rows_config2, rows_config3, weights_path
from gpu_helpers import oracle_model

pytestmark = pytest.mark.gpu
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _run(model, hb, dev, tap_rows=None):
    import torch
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    keep = [up(hb.tokens), up(hb.cu_seqlens), up(hb.mask_pos), up(hb.opt_off), up(hb.row_type)]
    b = jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)
    B, M, T = hb.n_rows, hb.n_markers, hb.n_tokens
    out = dict(logits=torch.empty(M, device=dev), probs=torch.empty(M, device=dev),
               choice=torch.empty(B, dtype=torch.int32, device=dev), score=torch.empty(B, device=dev),
               noul=torch.empty(B, device=dev), max_p=torch.empty(B, device=dev))
    taps = dict(encoder_out=torch.empty((T, 384), device=dev), marker_state=torch.empty((M, 384), device=dev))
    model.jd_decide(b, **out, taps=taps, stream=torch.cuda.current_stream())
    torch.cuda.synchronize()
    model.jd_check_status()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["marker_state"] = taps["marker_state"].cpu().numpy()
    enc = {}
    for i in tap_rows or []:
        s, e = int(hb.cu_seqlens[i]), int(hb.cu_seqlens[i + 1])
        enc[i] = taps["encoder_out"][s:e].cpu().numpy()
    return res, enc


def _check_row(hb, res, enc_rows, i, ref_logits, ref_hm, ref_enc, enc_pos=None, bf16=True):
    a, b = hb.opt_off[i], hb.opt_off[i + 1]
    z = res["logits"][a:b]
    ro = readouts(ref_logits, int(hb.row_type[i]))
    tl, tp, tr = (3e-2, 5e-3, 3e-2) if bf16 else (1e-3, 1e-4, 1e-4)
    assert np.abs(z - ref_logits).max() <= tl, (i, np.abs(z - ref_logits).max())
    assert np.abs(res["probs"][a:b] - ro["probs"]).max() <= tp
    srt = np.sort(ref_logits)[::-1]
    if srt[0] - srt[1] > 0.05:
        assert res["choice"][i] == ro["choice"]
    hm = res["marker_state"][a:b]
    assert np.linalg.norm(hm - ref_hm) / np.linalg.norm(ref_hm) <= tr
    e = enc_rows[i] if enc_pos is None else enc_rows[i][enc_pos]
    assert np.linalg.norm(e - ref_enc) / np.linalg.norm(ref_enc) <= tr
    return float(np.abs(z - ref_logits).max())


def test_throughput_full_size(weights_file):
    import torch
    from encoder_decision_model_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    rows = rows_config2(1024)
    opts = dict(max_length=1024, head_budget=512, strict=True)
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    lens = np.diff(hb.cu_seqlens)
    sample = sorted({0, 1, 511, 1023, int(lens.argmax()), int(lens.argmin())})
    model = jl.Model(weights_file, hb.n_tokens, hb.n_rows, hb.n_markers)
    res, enc = _run(model, hb, dev, tap_rows=sample)
    assert np.all(np.isfinite(res["logits"])) and np.all(np.isfinite(res["probs"]))
    # every row's probabilities sum to one
    sums = np.add.reduceat(res["probs"], hb.opt_off[:-1])
    np.testing.assert_allclose(sums, 1.0, atol=1e-5)
    om = oracle_model(str(weights_file))
    eo = EncodeOptions(max_length=1024, head_budget=512, strict=True)
    worst = 0.0
    for i in sample:
        r = om.forward_all(serialize_row(rows[i], eo))
        worst = max(worst, _check_row(hb, res, enc, i, r["logits"], r["marker_state"], r["encoder_out"]))
    print(f"throughput 1024 rows: sampled rows {sample}, max |delta logit| {worst:.2e}")
    # a row's result does not depend on its batch: the sampled rows scored alone (a batch of a few
    # row tiles, which takes the cluster-split residual GEMM) give the same logits bit for bit
    small = jl.Model(weights_file, 8192, 8, 256)
    for i in sample:
        alone = small.jd_decide_host([rows[i]], jl.encode_opts(**opts))
        a, b = hb.opt_off[i], hb.opt_off[i + 1]
        assert np.array_equal(alone["logits"], res["logits"][a:b]), (i, alone["logits"] - res["logits"][a:b])
    small.close()
    model.close()


@pytest.mark.parametrize("precision", [jl.JD_PREC_BF16, jl.JD_PREC_FP32])
def test_long_context_against_stored_oracle(weights_file, precision):
    import torch
    from encoder_decision_model_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    g = np.load(os.path.join(GOLD, "long_context_rows.npz"))
    rows = rows_config3(16)
    if precision == jl.JD_PREC_FP32:
        rows = [rows[i] for i in g["rows"]]  # the validation mode runs the two sampled rows only
        idx = {int(i): k for k, i in enumerate(g["rows"])}
    else:
        idx = {int(i): int(i) for i in g["rows"]}
    opts = dict(max_length=8192, head_budget=256, strict=False)
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    assert np.all(np.diff(hb.cu_seqlens) == 8192)
    model = jl.Model(weights_file, hb.n_tokens, hb.n_rows, hb.n_markers, precision=precision)
    res, enc = _run(model, hb, dev, tap_rows=list(idx.values()))
    for i, k in idx.items():
        d = _check_row(hb, res, enc, k, g[f"logits_{i}"], g[f"marker_state_{i}"], g[f"encoder_out_{i}"],
                       enc_pos=g[f"enc_pos_{i}"], bf16=precision == jl.JD_PREC_BF16)
        print(f"long context row {i} ({'bf16' if precision == 0 else 'fp32'}): max |delta logit| {d:.2e}")
    model.close()


def test_router_workload(weights_file):
    import torch
    from encoder_decision_model_b200.build import build
    build()
    dev = torch.device("cuda", 0)
    reqs = requests_config4(512)
    opts = jl.encode_opts(1024, 512, True)
    model = jl.Model(weights_file, 1 << 20, 2048, 2048 * 20)
    out = model.jd_route_host(reqs, opts)
    assert out["rows_per_round"].tolist() == [4 * 512, 512]  # 4 + 1 calls per request
    # for sampled requests: round 1 re-scored directly; the survivor rule on those
    # probabilities must give the final candidates, and the winner the final argmax
    om = oracle_model(str(weights_file))
    eo = EncodeOptions(max_length=1024, head_budget=512, strict=True)
    for r in (0, 137, 511):
        q = reqs[r]
        rows = [Row(state=q.state, question=q.question, options=q.labels[g:g + 20], qtype=0) for g in range(0, 72, 20)]
        ho = model.jd_decide_host(rows, opts)  # a row's result does not depend on its batch
        off = np.cumsum([0] + [len(x.options) for x in rows])
        expect = []
        for gi, g in enumerate(range(0, 72, 20)):
            expect += [g + k for k in survivors(ho["probs"][off[gi]:off[gi + 1]])]
        fc = out["final_candidates"][r]
        assert fc[fc >= 0].tolist() == expect
        fp = out["final_probs"][r][:len(expect)]
        assert out["winner"][r] == expect[int(np.argmax(fp))]
        np.testing.assert_allclose(fp.sum(), 1.0, atol=1e-5)
        # the final row's logits against the oracle
        final = Row(state=q.state, question=q.question, options=[q.labels[j] for j in expect], qtype=0)
        ref = om.logits(serialize_row(final, eo))
        hf = model.jd_decide_host([final], opts)
        assert np.abs(hf["logits"] - ref).max() <= 3e-2
        np.testing.assert_allclose(hf["probs"], fp, atol=1e-6)
        # round-1 logits of one group against the oracle
        ref1 = om.logits(serialize_row(rows[1], eo))
        assert np.abs(ho["logits"][off[1]:off[2]] - ref1).max() <= 3e-2
    model.close()
