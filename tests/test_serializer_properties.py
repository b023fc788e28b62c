"""Property-based check of the C serializer against the oracle's ("Julia-1: one
score per mask token", "From a state to one decision"): for any rows, budgets
and mode, either both succeed with bit-identical packed batches and encoding
reports, or both fail with the same status on the same row."""
import numpy as np
from hypothesis import HealthCheck, given, settings, strategies as st

from encoder_decision_model_b200 import _lib as jl
from oracle import EncodeOptions, EncodingError, serialize_row
from workloads import Row

ids = st.lists(st.integers(min_value=10, max_value=255999), max_size=70)


@st.composite
def rows(draw):
    qtype = draw(st.integers(0, 2))
    k = 2 if qtype == 2 and draw(st.booleans()) else draw(st.integers(1, 21))
    return Row(state=np.array(draw(st.lists(st.integers(10, 255999), max_size=300)), np.int32),
               question=np.array(draw(ids), np.int32),
               options=[np.array(draw(ids), np.int32) for _ in range(k)], qtype=qtype)


@settings(max_examples=300, deadline=None, suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(batch=st.lists(rows(), min_size=1, max_size=4), max_length=st.integers(1, 600),
       head_budget=st.integers(1, 600), strict=st.booleans())
def test_serializer_matches_oracle(batch, max_length, head_budget, strict):
    from encoder_decision_model_b200.build import build
    build()
    o = EncodeOptions(max_length=max_length, head_budget=head_budget, strict=strict)
    want, err = [], None
    for i, r in enumerate(batch):
        try:
            want.append(serialize_row(r, o))
        except EncodingError as e:
            err = (e.code, i)
            break
    opts = jl.encode_opts(max_length, head_budget, strict)
    try:
        hb = jl.jd_serialize(batch, opts)
    except jl.JDError as e:
        assert err == (e.code, e.bad_row)
        return
    assert err is None
    np.testing.assert_array_equal(hb.tokens, np.concatenate([e.ids for e in want]))
    cu = np.cumsum([0] + [len(e.ids) for e in want])
    np.testing.assert_array_equal(hb.cu_seqlens, cu)
    np.testing.assert_array_equal(hb.mask_pos, np.concatenate([e.mask_pos + cu[i] for i, e in enumerate(want)]))
    np.testing.assert_array_equal(hb.trunc, [e.trunc for e in want])
    np.testing.assert_array_equal(hb.head_len, [e.head_len for e in want])
    info = jl.jd_batch_info(hb)
    np.testing.assert_array_equal(info["length"], [len(e.ids) for e in want])
