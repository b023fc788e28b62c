"""Residual channels of magnitude ~4000 ("Julia-1 MLX", "Performance": the
residual stream stays in float32 because a few of its channels reach values
around 4000; the projections may run at lower precision).

Random weights do not grow such channels, so layer 0's Wo2 has four output rows
scaled so that those residual channels sit in the thousands from layer 0 to
the final norm.  Every later sublayer reads the residual through a LayerNorm,
whose statistics these channels then dominate: the other 380 channels of each
normalised row shrink by about 1/300.  The GPU path must keep both the large
channels and the shrunken ones: the encoder output's non-outlier channels are
held to the BF16 relative tolerance on their own, besides the usual logit,
probability and tap checks.
"""
import numpy as np
import pytest

from workloads import rows_config1, rows_config2, write_weights

CH = [5, 77, 200, 311]
SCALE = 6.0e4
OPT1 = dict(max_length=1024, head_budget=512, strict=True)


def _outlier_rows(a):
    a = a.copy()
    a[CH, :] *= SCALE
    return a


@pytest.fixture(scope="module")
def outlier_weights(tmp_path_factory):
    p = tmp_path_factory.mktemp("w") / "outlier.jdw"
    write_weights(p, seed=0, overrides={"enc.0.Wo2": _outlier_rows})
    return p


def test_outlier_channels_reach_thousands(outlier_weights):
    """The construction does what it claims, on the oracle: the four channels of
    the residual stay in the thousands through all 22 layers, the others near 1."""
    from oracle import OracleModel
    from oracle.model import encoder_layer, layer_norm
    from oracle.serialize import EncodeOptions, serialize_row

    m = OracleModel(outlier_weights)
    enc = serialize_row(rows_config1()[2], EncodeOptions(**OPT1))
    W, mo = m.W, m.mo
    x = layer_norm(W.embed_rows(enc.ids), W["embed.norm.g"], eps=mo.eps)
    others = np.delete(np.arange(x.shape[1]), CH)
    for l in range(mo.n_layers):
        x = encoder_layer(x, W, l, mo)
        big = np.abs(x[:, CH]).mean()
        assert 1000.0 < big < 10000.0, (l, big)
        assert np.abs(x[:, CH]).max() > 4000.0
        assert 0.5 < np.sqrt((x[:, others] ** 2).mean()) < 2.0


@pytest.mark.gpu
@pytest.mark.parametrize("precision", ["bf16", "fp32", "fp8"])
def test_outlier_residual_parity(outlier_weights, precision):
    """FP8 mode (E4M3 encoder QKV projections) is held to the BF16 bounds."""
    from encoder_decision_model_b200 import _lib as jl
    from encoder_decision_model_b200.build import build
    from gpu_helpers import compare, device_run, oracle_run

    build()
    bf16 = precision != "fp32"
    prec = {"bf16": jl.JD_PREC_BF16, "fp32": jl.JD_PREC_FP32, "fp8": jl.JD_PREC_FP8}[precision]
    m = jl.Model(outlier_weights, 16384, 64, 1024, precision=prec)
    rows = rows_config1() + rows_config2(4)
    hb, res = device_run(m, rows, OPT1, taps=True)
    ref = oracle_run(outlier_weights, rows, OPT1)
    compare(hb, res, ref, bf16=bf16, label=f"outlier {precision}")
    others = np.delete(np.arange(384), CH)
    tol = 3e-2 if bf16 else 1e-4
    for i, r in ref.items():
        s, e = hb.cu_seqlens[i], hb.cu_seqlens[i + 1]
        g = res["encoder_out"][s:e][:, others]
        o = r["encoder_out"][:, others]
        rel = np.linalg.norm(g - o) / np.linalg.norm(o)
        assert rel <= tol, (i, rel)
    m.close()
