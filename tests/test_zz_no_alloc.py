"""jd_forward_noalloc: the forward pass for callers that may not allocate
device memory while they run (for example a serving loop held to the budget it
reserved at start-up, or a host application that owns every device
allocation).  It keeps every intermediate in the library's static device
array.

What is checked, through the C ABI:
  * its logits equal jd_forward's bit for bit (the same kernels in the same
    launch configuration, on the same inputs), on consecutive calls that share
    the array, and match the oracle within the BF16 parity tolerance;
  * no call changes the device's free memory, the first one included
    (jd_model_create loads the array's module at start-up);
  * an id outside the vocabulary is reported by jd_noalloc_check_status, and a
    clean call after it reports nothing;
  * a batch beyond the stated maximum is refused with JD_ERR_CAPACITY.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import rows_config0, rows_config1

pytestmark = pytest.mark.gpu

TOL_LOGIT = 3e-2  # BF16 logit tolerance of the parity tests


def _device_batch(rows, opts, dev, tokens=None):
    import torch
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    keep = [up(hb.tokens) if tokens is None else tokens, up(hb.cu_seqlens), up(hb.mask_pos), up(hb.opt_off),
            up(hb.row_type)]
    return hb, keep, jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)


def test_forward_noalloc_matches_forward():
    import torch
    from encoder_decision_model_b200.build import build
    from gpu_helpers import oracle_run
    from workloads import weights_path

    build()
    assert torch.cuda.is_available()
    dev = torch.device("cuda", 0)
    wp = weights_path(0)
    model = jl.Model(wp, 4096, 16, 256, precision=jl.JD_PREC_BF16)
    o1 = dict(max_length=1024, head_budget=512, strict=True)
    o0 = dict(max_length=8192, head_budget=256, strict=True)
    cases = [(rows_config1(), o1), (rows_config0(), o0)]
    batches = [_device_batch(r, o, dev) for r, o in cases]
    ref = []
    for hb, keep, b in batches:
        z = torch.empty(hb.n_markers, device=dev)
        model.jd_forward(b, z)
        torch.cuda.synchronize()
        model.jd_check_status()
        ref.append(z.cpu().numpy())

    # the same 3-question batch with one id outside the vocabulary
    bad_tokens = batches[0][1][0].clone()
    bad_tokens[5] = 256000 + 7
    bad = _device_batch(rows_config1(), o1, dev, tokens=bad_tokens)
    outs = [torch.full((hb.n_markers,), float("nan"), device=dev) for hb, _, _ in batches]
    bad_out = torch.empty(bad[0].n_markers, device=dev)
    torch.cuda.synchronize()

    free0 = torch.cuda.mem_get_info(dev)[0]
    # two calls in a row on different batches, then the first batch again
    for i in (0, 1, 0):
        hb, keep, b = batches[i]
        outs[i].fill_(float("nan"))
        model.jd_forward_noalloc(b, outs[i])
        model.jd_noalloc_check_status()
        z = outs[i].cpu().numpy()
        assert np.all(np.isfinite(z))
        assert np.array_equal(z, ref[i]), f"batch {i}: max |delta logit| {np.abs(z - ref[i]).max()}"
        assert torch.cuda.mem_get_info(dev)[0] == free0, "device memory changed during the call"

    # an id outside the vocabulary: reported through the array's status word ...
    model.jd_forward_noalloc(bad[2], bad_out)
    with pytest.raises(jl.JDError) as ei:
        model.jd_noalloc_check_status()
    assert ei.value.code == jl.JD_ERR_DEVICE_STATUS
    # ... and cleared by the next call
    hb, keep, b = batches[1]
    model.jd_forward_noalloc(b, outs[1])
    model.jd_noalloc_check_status()
    assert np.array_equal(outs[1].cpu().numpy(), ref[1])
    assert torch.cuda.mem_get_info(dev)[0] == free0, "device memory changed during the calls"

    # against the oracle, at the parity tests' BF16 tolerance
    r1 = rows_config1()
    orc = oracle_run(wp, r1, o1)
    hb = batches[0][0]
    for i, r in orc.items():
        a, e = hb.opt_off[i], hb.opt_off[i + 1]
        d = float(np.abs(outs[0].cpu().numpy()[a:e] - r["logits"]).max())
        assert d <= TOL_LOGIT, f"row {i}: |delta logit| {d} against the oracle"

    # beyond the stated maximum: a clear error, no device work
    big = rows_config1() * 11
    hb, keep, b = _device_batch(big, o1, dev)
    assert hb.n_rows > 32
    with pytest.raises(jl.JDError) as ei:
        model.jd_forward_noalloc(b, torch.empty(hb.n_markers, device=dev))
    assert ei.value.code == jl.JD_ERR_CAPACITY
    model.close()
