"""CPU tests of the C ABI: exported symbols, the host serializer against the
oracle serializer (bit-exact) and loud failure without a CUDA device."""
import ctypes
import os
import re

import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from oracle import serialize_row, EncodeOptions, EncodingError
from workloads import Row, rows_config0, rows_config1, rows_config2, rows_config3, requests_config4, worked_example_rows

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from encoder_decision_model_b200.build import build
    build()
    return jl.lib()


def test_exports_every_declared_symbol(L):
    hdr = open(os.path.join(ROOT, "include", "julia_decide.h")).read()
    decls = "\n".join(l for l in hdr.splitlines() if not l.lstrip().startswith("typedef"))
    names = set(re.findall(r"\b(jd_[a-z_]+)\s*\(", decls))
    assert len(names) >= 13
    cdll = ctypes.CDLL(str(jl.LIB_PATH))
    missing = [n for n in sorted(names) if not hasattr(cdll, n)]
    assert not missing, missing


def _oracle_pack(rows, opt):
    encs = [serialize_row(r, opt) for r in rows]
    ids = np.concatenate([e.ids for e in encs])
    cu = np.cumsum([0] + [len(e.ids) for e in encs]).astype(np.int32)
    mp = np.concatenate([e.mask_pos + cu[i] for i, e in enumerate(encs)]).astype(np.int32)
    oo = np.cumsum([0] + [len(e.mask_pos) for e in encs]).astype(np.int32)
    return encs, ids, cu, mp, oo


def _compare(rows, max_length, head_budget, strict):
    o = EncodeOptions(max_length=max_length, head_budget=head_budget, strict=strict)
    encs, ids, cu, mp, oo = _oracle_pack(rows, o)
    hb = jl.jd_serialize(rows, jl.encode_opts(max_length, head_budget, strict))
    assert hb.n_rows == len(rows) and hb.n_tokens == len(ids) and hb.n_markers == len(mp)
    np.testing.assert_array_equal(hb.tokens, ids)
    np.testing.assert_array_equal(hb.cu_seqlens, cu)
    np.testing.assert_array_equal(hb.mask_pos, mp)
    np.testing.assert_array_equal(hb.opt_off, oo)
    np.testing.assert_array_equal(hb.row_type, [r.qtype for r in rows])
    np.testing.assert_array_equal(hb.trunc, [e.trunc for e in encs])
    np.testing.assert_array_equal(hb.head_len, [e.head_len for e in encs])
    assert hb.max_row_len == max(len(e.ids) for e in encs)


def test_serializer_configs_bit_exact(L):
    _compare(worked_example_rows(), 1024, 512, True)
    _compare(rows_config0(), 8192, 256, True)
    _compare(rows_config1(), 1024, 512, True)
    _compare(rows_config2(256), 1024, 512, True)
    _compare(rows_config3(4), 8192, 256, False)
    reqs = requests_config4(8)
    rows = [Row(state=r.state, question=r.question, options=r.labels[g:g + 20], qtype=0)
            for r in reqs for g in range(0, 72, 20)]
    _compare(rows, 1024, 512, True)


def _rand_rows(rng, n):
    rows = []
    for _ in range(n):
        k = int(rng.integers(2, 21))
        qtype = int(rng.integers(0, 3))
        if qtype == 2:
            k = 2
        rows.append(Row(state=rng.integers(10, 1000, size=int(rng.integers(0, 300))).astype(np.int32),
                        question=rng.integers(10, 1000, size=int(rng.integers(0, 40))).astype(np.int32),
                        options=[rng.integers(10, 1000, size=int(rng.integers(0, 70))).astype(np.int32)
                                 for _ in range(k)], qtype=qtype))
    return rows


def test_serializer_random_nonstrict_bit_exact(L):
    rng = np.random.default_rng(5)
    for budget, maxlen in ((64, 128), (40, 100), (256, 300), (30, 35), (512, 8192)):
        rows = _rand_rows(rng, 60)
        ok = []
        for r in rows:
            try:
                serialize_row(r, EncodeOptions(max_length=maxlen, head_budget=budget, strict=False))
                ok.append(r)
            except EncodingError:
                pass
        if ok:
            _compare(ok, maxlen, budget, False)


def test_serializer_error_codes_match_oracle(L):
    rng = np.random.default_rng(9)
    cases = []
    base = _rand_rows(rng, 1)[0]
    cases.append(Row(state=base.state, question=base.question, options=base.options[:1], qtype=0))
    cases.append(Row(state=base.state, question=base.question, options=[base.question] * 21, qtype=0))
    cases.append(Row(state=base.state, question=base.question, options=[base.question] * 3, qtype=2))
    bad = base.state.copy() if len(base.state) else np.array([5], np.int32)
    bad[0] = 256000
    cases.append(Row(state=bad, question=base.question, options=base.options, qtype=base.qtype))
    cases.append(Row(state=base.state, question=base.question, options=[np.arange(10, 60, dtype=np.int32)] * 2, qtype=1))
    cases.append(Row(state=np.arange(10, 2000, dtype=np.int32), question=base.question, options=base.options[:2], qtype=0))
    for strict in (True, False):
        for r in cases:
            o = EncodeOptions(max_length=512, head_budget=64, strict=strict)
            try:
                serialize_row(r, o)
                want = 0
            except EncodingError as e:
                want = e.code
            try:
                jl.jd_serialize([r], jl.encode_opts(512, 64, strict))
                got = 0
            except jl.JDError as e:
                got = e.code
                assert e.bad_row == 0
            assert got == want, (strict, got, want)


def test_serializer_reports_failing_row(L):
    rows = rows_config1()
    bad = Row(state=rows[0].state, question=rows[0].question, options=rows[0].options[:1], qtype=0)
    with pytest.raises(jl.JDError) as ei:
        jl.jd_serialize(rows + [bad], jl.encode_opts(1024, 512, True))
    assert ei.value.code == jl.JD_ERR_OPTION_COUNT and ei.value.bad_row == 3


def test_model_create_fails_loudly_without_gpu(L, weights_file):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(jl.JDError) as ei:
        jl.Model(weights_file, 1024, 4, 64)
    assert ei.value.code == jl.JD_ERR_CUDA


def test_version(L):
    assert "sm_100a" in jl.jd_version()


def test_shared_handle_argument_checks(L):
    cfg = jl.jd_model_config(1024, 8, 64, jl.JD_PREC_BF16, jl.JD_SCORER_MLP, jl.JD_ACT_RELU)
    h = ctypes.c_void_p()
    assert L.jd_model_create_shared(None, ctypes.byref(cfg), ctypes.byref(h)) == 1  # JD_ERR_INVALID_ARG
    assert not h.value


def test_marshalled_struct_layouts_match_ctypes():
    """The vectorised marshalling writes jd_row / jd_route_request records with numpy;
    their layout must be the C structures' (field offsets and size as ctypes lays them out)."""
    for ct in (jl.jd_row, jl.jd_route_request):
        dt = jl._struct_dtype(ct)
        assert dt.itemsize == ctypes.sizeof(ct)
        for name, typ in ct._fields_:
            assert dt.fields[name][1] == getattr(ct, name).offset, (ct.__name__, name)
            assert dt.fields[name][0].itemsize == ctypes.sizeof(typ), (ct.__name__, name)
    # a record written through numpy reads back field by field through ctypes
    rows = [Row(state=np.arange(5, 12), question=np.arange(20, 23), options=[np.arange(30, 34), np.arange(40, 42)], qtype=2)]
    keep = jl._RowKeep(rows)
    r = keep.arr[0]
    assert (r.n_state, r.n_question, r.k, r.type) == (7, 3, 2, 2)
    assert [r.state[i] for i in range(7)] == list(range(5, 12))
    assert [r.options[1][i] for i in range(r.n_option_ids[1])] == [40, 41]


@pytest.mark.parametrize("field", ["bos", "eos", "mask"])
@pytest.mark.parametrize("value", [-1, 256000])
def test_special_ids_out_of_range(L, field, value):
    """A special id outside [0, vocab) is rejected like any other id, by the C
    serializer and the oracle alike; it is an options error, so no row is blamed."""
    rows = rows_config1()
    kw = dict(bos=2, eos=1, mask=4)
    kw[field] = value
    with pytest.raises(EncodingError) as eo:
        serialize_row(rows[0], EncodeOptions(max_length=1024, head_budget=512, strict=True, **kw))
    with pytest.raises(jl.JDError) as ei:
        jl.jd_serialize(rows, jl.encode_opts(1024, 512, True, **kw))
    assert ei.value.code == eo.value.code == jl.JD_ERR_TOKEN_RANGE
    assert ei.value.bad_row == -1


def test_null_arrays_with_zero_lengths(L):
    """Empty question, state and option arrays may be passed as NULL pointers."""
    i32p = ctypes.POINTER(ctypes.c_int32)
    opt0 = np.array([11, 12, 13], np.int32)
    optp = (i32p * 2)(opt0.ctypes.data_as(i32p), i32p())
    optn = (ctypes.c_int32 * 2)(3, 0)
    row = jl.jd_row()
    row.state, row.n_state = None, 0
    row.question, row.n_question = None, 0
    row.options = ctypes.cast(optp, type(row.options))
    row.n_option_ids = ctypes.cast(optn, type(row.n_option_ids))
    row.k, row.type = 2, 0
    out = ctypes.POINTER(jl.jd_batch)()
    bad = ctypes.c_int32(-1)
    opts = jl.encode_opts(64, 64, True)
    assert L.jd_serialize(ctypes.byref(row), 1, ctypes.byref(opts), ctypes.byref(out), ctypes.byref(bad)) == 0
    b = out.contents
    toks = np.ctypeslib.as_array(ctypes.cast(b.tokens, i32p), shape=(b.n_tokens,)).copy()
    mp = np.ctypeslib.as_array(ctypes.cast(b.mask_pos, i32p), shape=(b.n_markers,)).copy()
    L.jd_batch_free(out)
    enc = serialize_row(Row(state=np.zeros(0, np.int32), question=np.zeros(0, np.int32),
                            options=[opt0, np.zeros(0, np.int32)], qtype=0),
                        EncodeOptions(max_length=64, head_budget=64, strict=True))
    np.testing.assert_array_equal(toks, enc.ids)
    np.testing.assert_array_equal(mp, enc.mask_pos)


def test_route_requires_winner_output(L):
    """jd_route_host checks its arguments before it touches the model: a NULL
    winner array is JD_ERR_INVALID_ARG (the handle here is a dummy host buffer
    that the call never reaches)."""
    i32p = ctypes.POINTER(ctypes.c_int32)
    lab = np.array([10, 11], np.int32)
    labp = (i32p * 3)(*([lab.ctypes.data_as(i32p)] * 3))
    labn = (ctypes.c_int32 * 3)(2, 2, 2)
    st = np.arange(10, 20, dtype=np.int32)
    req = jl.jd_route_request()
    req.state, req.n_state = st.ctypes.data_as(i32p), len(st)
    req.question, req.n_question = None, 0
    req.labels = ctypes.cast(labp, type(req.labels))
    req.n_label_ids = ctypes.cast(labn, type(req.n_label_ids))
    req.n_labels = 3
    out = jl.jd_route_outputs()
    dummy = ctypes.create_string_buffer(64)
    opts = jl.encode_opts(1024, 512, True)
    code = L.jd_route_host(ctypes.cast(dummy, ctypes.c_void_p), ctypes.byref(req), 1, ctypes.byref(opts),
                           4096, 16, 64, ctypes.byref(out), None)
    assert code == jl.JD_ERR_INVALID_ARG
    assert "winner" in L.jd_last_error().decode()


def _oracle_info(rows, opt):
    out = {k: [] for k in jl.ENCODING_INFO_FIELDS}
    for r in rows:
        e = serialize_row(r, opt)
        out["length"].append(len(e.ids))
        out["head_length"].append(e.head_len)
        out["state_length"].append(len(e.ids) - e.head_len - 1)
        out["n_options"].append(len(e.mask_pos))
        out["truncated"].append(e.trunc)
    return out


@pytest.mark.parametrize("case", ["c1", "c2", "c3", "random"])
def test_encoding_info_matches_oracle(L, case):
    """The encoding_info report ("Julia-1 MLX", "API"), from rows and from a host
    batch, against the oracle serializer row by row."""
    if case == "c1":
        rows, args = rows_config1(), (1024, 512, True)
    elif case == "c2":
        rows, args = rows_config2(64), (1024, 512, True)
    elif case == "c3":
        rows, args = rows_config3(4), (8192, 256, False)
    else:
        rng = np.random.default_rng(21)
        rows, args = [], (128, 64, False)
        for r in _rand_rows(rng, 80):
            try:
                serialize_row(r, EncodeOptions(max_length=128, head_budget=64, strict=False))
                rows.append(r)
            except EncodingError:
                pass
    want = _oracle_info(rows, EncodeOptions(max_length=args[0], head_budget=args[1], strict=args[2]))
    got = jl.jd_rows_encoding_info(rows, jl.encode_opts(*args))
    got_b = jl.jd_batch_info(jl.jd_serialize(rows, jl.encode_opts(*args)))
    for k in jl.ENCODING_INFO_FIELDS:
        np.testing.assert_array_equal(got[k], want[k], err_msg=k)
        np.testing.assert_array_equal(got_b[k], want[k], err_msg=k)
    if case in ("c3", "random"):
        assert any(want["truncated"]), "the non-strict cases must exercise truncation"


def test_encoding_info_errors(L):
    rows = rows_config1()
    bad = Row(state=rows[0].state, question=rows[0].question, options=rows[0].options[:1], qtype=0)
    with pytest.raises(jl.JDError) as ei:
        jl.jd_rows_encoding_info(rows + [bad], jl.encode_opts(1024, 512, True))
    assert ei.value.code == jl.JD_ERR_OPTION_COUNT and ei.value.bad_row == 3
    # a device-style batch (no host-side head_len / trunc) is refused
    hb = jl.jd_serialize(rows, jl.encode_opts(1024, 512, True))
    bs = hb.as_struct()
    bs.head_len = None
    out = np.zeros((len(rows), 5), np.int32)
    assert L.jd_batch_info(ctypes.byref(bs), out.ctypes.data) == jl.JD_ERR_INVALID_ARG
