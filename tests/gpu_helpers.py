"""Shared helpers of the GPU parity tests: run the library through its C ABI on
torch-allocated device buffers, and the oracle on the same rows."""
from __future__ import annotations

import functools

import numpy as np

from encoder_decision_model_b200 import _lib as jl
from oracle import EncodeOptions, OracleModel, ModelOptions, serialize_row


def device_run(model, rows, opts, taps=False, stream=None):
    """Serialize with the C serializer, upload, run jd_decide; numpy results."""
    import torch

    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    dev = torch.device("cuda")

    def up(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    tokens, cu, mp, oo, rt = up(hb.tokens), up(hb.cu_seqlens), up(hb.mask_pos), up(hb.opt_off), up(hb.row_type)
    batch = jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, tokens, cu, mp, oo, rt)
    B, M, T = hb.n_rows, hb.n_markers, hb.n_tokens
    out = dict(logits=torch.full((M,), float("nan"), device=dev), probs=torch.full((M,), float("nan"), device=dev),
               choice=torch.full((B,), -1, dtype=torch.int32, device=dev), score=torch.empty(B, device=dev),
               noul=torch.empty(B, device=dev), max_p=torch.empty(B, device=dev))
    tp = None
    if taps:
        tp = dict(encoder_out=torch.full((T, 384), float("nan"), device=dev),
                  marker_state=torch.full((M, 384), float("nan"), device=dev))
    st = stream or torch.cuda.current_stream()
    model.jd_decide(batch, **out, taps=tp, stream=st)
    torch.cuda.synchronize()
    model.jd_check_status()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    if tp:
        res.update({k: v.cpu().numpy() for k, v in tp.items()})
    res["_keep"] = (tokens, cu, mp, oo, rt)
    return hb, res


@functools.lru_cache(maxsize=None)
def oracle_model(path, scorer="mlp", head_act="relu"):
    return OracleModel(path, ModelOptions(scorer=scorer, head_act=head_act))


def oracle_run(path, rows, opts, scorer="mlp", head_act="relu", row_ids=None):
    """Oracle results per row: list of dicts (encoder_out, marker_state, logits)."""
    m = oracle_model(str(path), scorer, head_act)
    eo = EncodeOptions(max_length=opts["max_length"], head_budget=opts["head_budget"], strict=opts["strict"])
    idx = range(len(rows)) if row_ids is None else row_ids
    return {i: m.forward_all(serialize_row(rows[i], eo)) for i in idx}


def compare(hb, res, ref, bf16, check_taps=True, label=""):
    """Assert the parity tolerances row by row; returns summary stats."""
    from oracle import readouts

    worst = dict(logit=0.0, prob=0.0, enc_rel=0.0, hm_rel=0.0, argmax_checked=0, spread=0.0)
    for i, r in ref.items():
        a, b = hb.opt_off[i], hb.opt_off[i + 1]
        z = res["logits"][a:b]
        zr = r["logits"]
        assert np.all(np.isfinite(z)), f"{label} row {i}: non-finite logits"
        d = np.abs(z - zr).max()
        worst["logit"] = max(worst["logit"], d)
        worst["spread"] = max(worst["spread"], float(zr.max() - zr.min()))
        ro = readouts(zr, int(hb.row_type[i]))
        dp = np.abs(res["probs"][a:b] - ro["probs"]).max()
        worst["prob"] = max(worst["prob"], dp)
        srt = np.sort(zr)[::-1]
        if srt[0] - srt[1] > 0.05:
            worst["argmax_checked"] += 1
            assert res["choice"][i] == ro["choice"], f"{label} row {i}: argmax differs with gap {srt[0] - srt[1]:.3f}"
        assert abs(res["score"][i] - ro["score"]) <= (5e-3 * (b - a) if bf16 else 1e-4 * (b - a))
        if hb.row_type[i] == 2:
            assert abs(res["noul"][i] - ro["noul"]) <= (5e-3 if bf16 else 1e-4)
        else:
            assert np.isnan(res["noul"][i])
        assert abs(res["max_p"][i] - ro["max_p"]) <= (5e-3 if bf16 else 1e-4)
        if check_taps and "encoder_out" in res:
            s, e = hb.cu_seqlens[i], hb.cu_seqlens[i + 1]
            ge = res["encoder_out"][s:e]
            rel = np.linalg.norm(ge - r["encoder_out"]) / np.linalg.norm(r["encoder_out"])
            worst["enc_rel"] = max(worst["enc_rel"], rel)
            gh = res["marker_state"][a:b]
            relh = np.linalg.norm(gh - r["marker_state"]) / np.linalg.norm(r["marker_state"])
            worst["hm_rel"] = max(worst["hm_rel"], relh)
    tol_logit = 3e-2 if bf16 else 1e-3
    tol_prob = 5e-3 if bf16 else 1e-4
    tol_rel = 3e-2 if bf16 else 1e-4
    msg = f"{label}: {worst}"
    assert worst["logit"] <= tol_logit, msg
    assert worst["prob"] <= tol_prob, msg
    assert worst["enc_rel"] <= tol_rel and worst["hm_rel"] <= tol_rel, msg
    print(msg)
    return worst
