"""jd_forward_noalloc: the forward pass for callers that may not allocate
device memory while they run (for example a serving loop held to the budget it
reserved at start-up).  It keeps every intermediate in the library's static
device array; its logits must match jd_forward's within the BF16 tolerance of
the parity tests, on consecutive calls that share that array.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import rows_config0, rows_config1

pytestmark = pytest.mark.gpu

TOL_LOGIT = 3e-2  # BF16 logit tolerance of the parity tests


def _device_batch(rows, opts, dev):
    import torch
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    keep = [up(hb.tokens), up(hb.cu_seqlens), up(hb.mask_pos), up(hb.opt_off), up(hb.row_type)]
    return hb, keep, jl.Model.device_batch(hb.n_rows, hb.n_tokens, hb.n_markers, hb.max_row_len, *keep)


def test_forward_noalloc_matches_forward():
    import torch
    from encoder_decision_model_b200.build import build
    from workloads import weights_path

    build()
    assert torch.cuda.is_available()
    dev = torch.device("cuda", 0)
    model = jl.Model(weights_path(0), 4096, 16, 256, precision=jl.JD_PREC_BF16)
    cases = [(rows_config1(), dict(max_length=1024, head_budget=512, strict=True)),
             (rows_config0(), dict(max_length=8192, head_budget=256, strict=True))]
    batches = [_device_batch(r, o, dev) for r, o in cases]
    ref = []
    for hb, keep, b in batches:
        z = torch.empty(hb.n_markers, device=dev)
        model.jd_forward(b, z)
        torch.cuda.synchronize()
        model.jd_check_status()
        ref.append(z.cpu().numpy())
    outs = [torch.full((hb.n_markers,), float("nan"), device=dev) for hb, _, _ in batches]
    # two calls in a row on different batches, then the first batch again
    for k, i in enumerate((0, 1, 0)):
        hb, keep, b = batches[i]
        # after the first call (which may load the library's device module) no call changes free memory
        free0 = torch.cuda.mem_get_info(dev)[0] if k > 0 else None
        model.jd_forward_noalloc(b, outs[i])
        torch.cuda.synchronize()
        z = outs[i].cpu().numpy()
        assert np.all(np.isfinite(z))
        d = float(np.abs(z - ref[i]).max())
        assert d <= TOL_LOGIT, f"batch {i}: max |delta logit| {d}"
        if free0 is not None:
            assert torch.cuda.mem_get_info(dev)[0] == free0, "device memory changed during the call"
    # beyond the stated maximum: a clear error, no device work
    big = rows_config1() * 11
    hb, keep, b = _device_batch(big, dict(max_length=1024, head_budget=512, strict=True), dev)
    assert hb.n_rows > 32
    with pytest.raises(jl.JDError) as ei:
        model.jd_forward_noalloc(b, torch.empty(hb.n_markers, device=dev))
    assert ei.value.code == jl.JD_ERR_CAPACITY
    model.close()
