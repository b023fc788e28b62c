"""ctypes binding of libjulia_decide.so (argument marshalling only).

Every function here forwards to the C entry point of the same name declared in
include/julia_decide.h; no step of the forward pass runs in Python.  Device
buffers are passed as integers or objects with a ``data_ptr()`` method (torch
tensors); streams as integers or objects with a ``cuda_stream`` attribute.
"""
from __future__ import annotations

import ctypes as C
import os
from pathlib import Path

import numpy as np

LIB_PATH = Path(__file__).resolve().parent / "libjulia_decide.so"

JD_OK, JD_ERR_INVALID_ARG, JD_ERR_OPTION_COUNT, JD_ERR_OVERFLOW, JD_ERR_TOKEN_RANGE = 0, 1, 2, 3, 4
JD_ERR_CAPACITY, JD_ERR_CUDA, JD_ERR_DEVICE_STATUS, JD_ERR_IO = 5, 6, 7, 8
JD_PREC_BF16, JD_PREC_FP32, JD_PREC_FP8 = 0, 1, 2
JD_SCORER_MLP, JD_SCORER_LINEAR = 0, 1
JD_ACT_RELU, JD_ACT_GELU = 0, 1

i32p = C.POINTER(C.c_int32)
f32p = C.POINTER(C.c_float)


class jd_row(C.Structure):
    _fields_ = [("state", i32p), ("n_state", C.c_int32), ("question", i32p), ("n_question", C.c_int32),
                ("options", C.POINTER(i32p)), ("n_option_ids", i32p), ("k", C.c_int32), ("type", C.c_int32)]


class jd_encode_opts(C.Structure):
    _fields_ = [("max_length", C.c_int32), ("head_budget", C.c_int32), ("strict", C.c_int32),
                ("bos", C.c_int32), ("eos", C.c_int32), ("mask", C.c_int32), ("vocab", C.c_int32)]


class jd_batch(C.Structure):
    _fields_ = [("n_rows", C.c_int32), ("n_tokens", C.c_int32), ("n_markers", C.c_int32),
                ("max_row_len", C.c_int32), ("tokens", C.c_void_p), ("cu_seqlens", C.c_void_p),
                ("mask_pos", C.c_void_p), ("opt_off", C.c_void_p), ("row_type", C.c_void_p),
                ("head_len", C.c_void_p), ("trunc", C.c_void_p)]


class jd_outputs(C.Structure):
    _fields_ = [("logits", C.c_void_p), ("probs", C.c_void_p), ("choice", C.c_void_p), ("score", C.c_void_p),
                ("noul", C.c_void_p), ("max_p", C.c_void_p)]


class jd_taps(C.Structure):
    _fields_ = [("encoder_out", C.c_void_p), ("marker_state", C.c_void_p)]


class jd_model_config(C.Structure):
    _fields_ = [("max_tokens", C.c_int32), ("max_rows", C.c_int32), ("max_markers", C.c_int32),
                ("precision", C.c_int32), ("scorer", C.c_int32), ("head_act", C.c_int32)]


class jd_host_outputs(C.Structure):
    _fields_ = [("logits", f32p), ("probs", f32p), ("choice", i32p), ("score", f32p), ("noul", f32p),
                ("max_p", f32p), ("n_rows", C.c_int32), ("n_markers", C.c_int32)]


class jd_route_request(C.Structure):
    _fields_ = [("state", i32p), ("n_state", C.c_int32), ("question", i32p), ("n_question", C.c_int32),
                ("labels", C.POINTER(i32p)), ("n_label_ids", i32p), ("n_labels", C.c_int32)]


class jd_route_outputs(C.Structure):
    _fields_ = [("winner", i32p), ("winner_p", f32p), ("final_candidates", i32p), ("final_probs", f32p),
                ("rows_per_round", i32p), ("max_rounds", C.c_int32), ("n_rounds", C.c_int32)]


# jd_route_scorer: (user, rows, n_rows, probs) -> jd_status
ROUTE_SCORER = C.CFUNCTYPE(C.c_int, C.c_void_p, C.POINTER(jd_row), C.c_int32, C.POINTER(C.c_float))


class JDError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"[{code}] {msg}")
        self.code = code


_lib = None


def lib():
    """Load the CUDA library; raises if it has not been built (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    path = Path(os.environ.get("JD_LIB", LIB_PATH))
    if not path.exists():
        raise FileNotFoundError(f"{path} is missing: build it with python -m encoder_decision_model_b200.build")
    L = C.CDLL(str(path))
    L.jd_last_error.restype = C.c_char_p
    L.jd_version.restype = C.c_char_p
    L.jd_serialize.argtypes = [C.POINTER(jd_row), C.c_int32, C.POINTER(jd_encode_opts),
                               C.POINTER(C.POINTER(jd_batch)), C.POINTER(C.c_int32)]
    L.jd_batch_free.argtypes = [C.POINTER(jd_batch)]
    L.jd_batch_free.restype = None
    L.jd_batch_info.argtypes = [C.POINTER(jd_batch), C.c_void_p]
    L.jd_route_scored.argtypes = [C.POINTER(jd_route_request), C.c_int32, ROUTE_SCORER, C.c_void_p,
                                  C.POINTER(jd_route_outputs)]
    L.jd_rows_encoding_info.argtypes = [C.POINTER(jd_row), C.c_int32, C.POINTER(jd_encode_opts), C.c_void_p,
                                        C.POINTER(C.c_int32)]
    L.jd_model_create.argtypes = [C.POINTER(jd_model_config), C.c_char_p, C.c_int, C.POINTER(C.c_void_p)]
    L.jd_model_create_shared.argtypes = [C.c_void_p, C.POINTER(jd_model_config), C.POINTER(C.c_void_p)]
    L.jd_model_destroy.argtypes = [C.c_void_p]
    L.jd_model_destroy.restype = None
    L.jd_model_device_bytes.argtypes = [C.c_void_p]
    L.jd_model_device_bytes.restype = C.c_size_t
    L.jd_decide.argtypes = [C.c_void_p, C.POINTER(jd_batch), C.POINTER(jd_outputs), C.POINTER(jd_taps), C.c_void_p]
    L.jd_forward.argtypes = [C.c_void_p, C.POINTER(jd_batch), C.c_void_p, C.c_void_p]
    L.jd_decide_host.argtypes = [C.c_void_p, C.POINTER(jd_row), C.c_int32, C.POINTER(jd_encode_opts),
                                 C.POINTER(jd_host_outputs), C.c_void_p]
    L.jd_decide_packed_host.argtypes = [C.c_void_p, C.POINTER(jd_batch), C.POINTER(jd_host_outputs), C.c_void_p]
    L.jd_decide_host_submit.argtypes = [C.c_void_p, C.POINTER(jd_row), C.c_int32, C.POINTER(jd_encode_opts),
                                        C.c_void_p, C.POINTER(C.c_int64)]
    L.jd_decide_host_submit.restype = C.c_int
    L.jd_decide_host_collect.argtypes = [C.c_void_p, C.c_int64, C.POINTER(jd_host_outputs)]
    L.jd_decide_host_collect.restype = C.c_int
    L.jd_check_status.argtypes = [C.c_void_p]
    L.jd_set_graph_mode.argtypes = [C.c_void_p, C.c_int]
    L.jd_graph_stats.argtypes = [C.c_void_p, C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int32)]
    L.jd_route_host.argtypes = [C.c_void_p, C.POINTER(jd_route_request), C.c_int32, C.POINTER(jd_encode_opts),
                                C.c_int32, C.c_int32, C.c_int32, C.POINTER(jd_route_outputs), C.c_void_p]
    L.jd_route_host.restype = C.c_int
    L.jd_route_device.argtypes = [C.c_void_p, C.POINTER(jd_route_request), C.c_int32, C.POINTER(jd_encode_opts),
                                  C.POINTER(jd_route_outputs), C.c_void_p]
    L.jd_route_device.restype = C.c_int
    L.jd_forward_noalloc.argtypes = [C.c_void_p, C.POINTER(jd_batch), C.c_void_p, C.c_void_p]
    L.jd_forward_noalloc.restype = C.c_int
    L.jd_noalloc_check_status.argtypes = [C.c_void_p, C.c_void_p]
    L.jd_noalloc_check_status.restype = C.c_int
    L.jd_last_launch_count.argtypes = [C.c_void_p]
    L.jd_last_launch_count.restype = C.c_int32
    L.jd_set_profiling.argtypes = [C.c_void_p, C.c_int]
    L.jd_profile_report.argtypes = [C.c_void_p, C.c_char_p, C.c_size_t]
    for name in ("jd_serialize", "jd_model_create", "jd_model_create_shared", "jd_decide", "jd_forward", "jd_decide_host",
                 "jd_decide_packed_host", "jd_check_status", "jd_set_graph_mode", "jd_graph_stats", "jd_set_profiling",
                 "jd_profile_report"):
        getattr(L, name).restype = C.c_int
    _lib = L
    return L


def _check(code):
    if code != JD_OK:
        raise JDError(code, lib().jd_last_error().decode())


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        return x.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def jd_version():
    return lib().jd_version().decode()


def encode_opts(max_length=8192, head_budget=256, strict=True, bos=2, eos=1, mask=4, vocab=256000):
    return jd_encode_opts(max_length, head_budget, int(bool(strict)), bos, eos, mask, vocab)


def _struct_dtype(ct):
    """numpy dtype with the byte layout of ctypes structure `ct` (pointers as uint64)."""
    names, formats, offsets = [], [], []
    for name, typ in ct._fields_:
        names.append(name)
        formats.append(np.int32 if typ is C.c_int32 else np.uint64)
        offsets.append(getattr(ct, name).offset)
    return np.dtype({"names": names, "formats": formats, "offsets": offsets, "itemsize": C.sizeof(ct)})


def _pack_lists(seqs):
    """One int32 buffer for a list of id sequences: (flat, offsets, lengths)."""
    lens = np.fromiter((len(x) for x in seqs), dtype=np.int64, count=len(seqs))
    flat = np.concatenate([np.asarray(x, dtype=np.int32).ravel() for x in seqs]) if seqs else np.zeros(0, np.int32)
    flat = np.ascontiguousarray(flat, dtype=np.int32)
    offs = np.zeros(len(seqs), dtype=np.int64)
    if len(seqs) > 1:
        np.cumsum(lens[:-1], out=offs[1:])
    return flat, offs, lens


class _RowKeep:
    """The jd_row array of `rows` and the buffers it points into, built with
    vectorised numpy (one buffer per field kind, not one object per option)."""

    def __init__(self, rows):
        n = len(rows)
        st, st_off, st_len = _pack_lists([r.state for r in rows])
        q, q_off, q_len = _pack_lists([r.question for r in rows])
        k = np.fromiter((len(r.options) for r in rows), dtype=np.int64, count=n)
        opt, o_off, o_len = _pack_lists([o for r in rows for o in r.options])
        optp = (opt.ctypes.data + 4 * o_off).astype(np.uint64) if len(o_off) else np.zeros(1, np.uint64)
        olen = o_len.astype(np.int32) if len(o_len) else np.zeros(1, np.int32)
        first = np.zeros(n, dtype=np.int64)
        if n > 1:
            np.cumsum(k[:-1], out=first[1:])
        arr = np.zeros(max(1, n), dtype=_struct_dtype(jd_row))
        if n:
            arr["state"][:n] = st.ctypes.data + 4 * st_off
            arr["n_state"][:n] = st_len
            arr["question"][:n] = q.ctypes.data + 4 * q_off
            arr["n_question"][:n] = q_len
            arr["options"][:n] = optp.ctypes.data + 8 * first
            arr["n_option_ids"][:n] = olen.ctypes.data + 4 * first
            arr["k"][:n] = k
            arr["type"][:n] = np.fromiter((int(r.qtype) for r in rows), dtype=np.int32, count=n)
        self.keep = (st, q, opt, optp, olen, arr)
        self.arr = arr.ctypes.data_as(C.POINTER(jd_row))


class HostBatch:
    """A packed batch copied out of jd_serialize into numpy arrays."""

    def __init__(self, d):
        self.__dict__.update(d)

    def as_struct(self):
        """jd_batch over these host arrays (kept alive by self)."""
        return jd_batch(self.n_rows, self.n_tokens, self.n_markers, self.max_row_len, self.tokens.ctypes.data,
                        self.cu_seqlens.ctypes.data, self.mask_pos.ctypes.data, self.opt_off.ctypes.data,
                        self.row_type.ctypes.data, self.head_len.ctypes.data, self.trunc.ctypes.data)


def jd_serialize(rows, opts: jd_encode_opts):
    """Serialize rows (objects with state/question/options/qtype) -> HostBatch.

    Raises JDError with the C status code; the failing row index is in
    ``err.bad_row``.
    """
    L = lib()
    keep = _RowKeep(rows)
    out = C.POINTER(jd_batch)()
    bad = C.c_int32(-1)
    code = L.jd_serialize(keep.arr, len(rows), C.byref(opts), C.byref(out), C.byref(bad))
    if code != JD_OK:
        e = JDError(code, L.jd_last_error().decode())
        e.bad_row = bad.value
        raise e
    b = out.contents

    def arr(ptr, n, dt):
        if n == 0:
            return np.zeros(0, dt)
        ct = C.c_int32 if dt == np.int32 else C.c_uint8
        return np.ctypeslib.as_array(C.cast(ptr, C.POINTER(ct)), shape=(n,)).copy()

    d = dict(n_rows=b.n_rows, n_tokens=b.n_tokens, n_markers=b.n_markers, max_row_len=b.max_row_len,
             tokens=arr(b.tokens, b.n_tokens, np.int32), cu_seqlens=arr(b.cu_seqlens, b.n_rows + 1, np.int32),
             mask_pos=arr(b.mask_pos, b.n_markers, np.int32), opt_off=arr(b.opt_off, b.n_rows + 1, np.int32),
             row_type=arr(b.row_type, b.n_rows, np.int32), head_len=arr(b.head_len, b.n_rows, np.int32),
             trunc=arr(b.trunc, b.n_rows, np.uint8))
    L.jd_batch_free(out)
    return HostBatch(d)


# jd_encoding_info fields, in order (five int32 per row)
ENCODING_INFO_FIELDS = ("length", "head_length", "state_length", "n_options", "truncated")


def _info_dict(a):
    return {k: a[:, i].copy() for i, k in enumerate(ENCODING_INFO_FIELDS)}


def jd_rows_encoding_info(rows, opts: jd_encode_opts):
    """Per-row encoding report of `rows` (jd_rows_encoding_info): dict of int32
    arrays keyed by ENCODING_INFO_FIELDS.  Raises JDError like jd_serialize."""
    keep = _RowKeep(rows)
    a = np.zeros((max(1, len(rows)), len(ENCODING_INFO_FIELDS)), np.int32)
    bad = C.c_int32(-1)
    code = lib().jd_rows_encoding_info(keep.arr, len(rows), C.byref(opts), a.ctypes.data, C.byref(bad))
    if code != JD_OK:
        e = JDError(code, lib().jd_last_error().decode())
        e.bad_row = bad.value
        raise e
    return _info_dict(a[:len(rows)])


def jd_batch_info(hb: HostBatch):
    """Per-row encoding report of a serialized host batch (jd_batch_info)."""
    a = np.zeros((max(1, hb.n_rows), len(ENCODING_INFO_FIELDS)), np.int32)
    bs = hb.as_struct()
    _check(lib().jd_batch_info(C.byref(bs), a.ctypes.data))
    return _info_dict(a[:hb.n_rows])


def _route_marshal(requests):
    """jd_route_request records for `requests` (objects with state/question/labels),
    the arrays they point into, and the outputs dict with its jd_route_outputs."""
    n = len(requests)
    st, st_off, st_len = _pack_lists([r.state for r in requests])
    q, q_off, q_len = _pack_lists([r.question for r in requests])
    nl = np.fromiter((len(r.labels) for r in requests), dtype=np.int64, count=n)
    lab, l_off, l_len = _pack_lists([x for r in requests for x in r.labels])
    labp = (lab.ctypes.data + 4 * l_off).astype(np.uint64) if len(l_off) else np.zeros(1, np.uint64)
    llen = l_len.astype(np.int32) if len(l_len) else np.zeros(1, np.int32)
    first = np.zeros(n, dtype=np.int64)
    if n > 1:
        np.cumsum(nl[:-1], out=first[1:])
    req = np.zeros(max(1, n), dtype=_struct_dtype(jd_route_request))
    if n:
        req["state"][:n] = st.ctypes.data + 4 * st_off
        req["n_state"][:n] = st_len
        req["question"][:n] = q.ctypes.data + 4 * q_off
        req["n_question"][:n] = q_len
        req["labels"][:n] = labp.ctypes.data + 8 * first
        req["n_label_ids"][:n] = llen.ctypes.data + 4 * first
        req["n_labels"][:n] = nl
    keep = (st, q, lab, labp, llen, req)
    arr = req.ctypes.data_as(C.POINTER(jd_route_request))
    o = dict(winner=np.zeros(n, np.int32), winner_p=np.zeros(n, np.float32),
             final_candidates=np.zeros((n, 20), np.int32), final_probs=np.zeros((n, 20), np.float32),
             rows_per_round=np.zeros(16, np.int32))
    s = jd_route_outputs(o["winner"].ctypes.data_as(i32p), o["winner_p"].ctypes.data_as(f32p),
                         o["final_candidates"].ctypes.data_as(i32p), o["final_probs"].ctypes.data_as(f32p),
                         o["rows_per_round"].ctypes.data_as(i32p), 16, 0)
    return arr, keep, o, s


def _route_result(o, s):
    o["rows_per_round"] = o["rows_per_round"][:s.n_rounds]
    return o


def jd_route_scored(requests, score):
    """The Router's tournament (jd_route_scored) with `score` as the scorer:
    score(rows) gets, per row, the list of its options' label-id arrays and
    returns, per row, the option probabilities (float32 is what the library
    keeps).  Returns the same dict as Model.jd_route_host."""
    arr, keep, o, s = _route_marshal(requests)
    err = []

    def cb(user, rows, n_rows, probs):
        try:
            opts = []
            for i in range(n_rows):
                r = rows[i]
                opts.append([np.ctypeslib.as_array(r.options[k], shape=(r.n_option_ids[k],)).copy()
                             if r.n_option_ids[k] else np.zeros(0, np.int32) for k in range(r.k)])
            ps = score(opts)
            flat = np.concatenate([np.asarray(p, np.float32) for p in ps])
            if len(flat) != sum(len(x) for x in opts):
                raise ValueError("score() returned the wrong number of probabilities")
            C.memmove(probs, flat.ctypes.data, flat.nbytes)
            return JD_OK
        except Exception as e:  # reported after the call; the library sees a failed status
            err.append(e)
            return JD_ERR_INVALID_ARG

    fn = ROUTE_SCORER(cb)
    code = lib().jd_route_scored(arr, len(requests), fn, None, C.byref(s))
    if err:
        raise err[0]
    _check(code)
    return _route_result(o, s)


class Model:
    """Owner of a jd_model handle (weights + workspace on one device)."""

    def __init__(self, weights_path, max_tokens, max_rows, max_markers, precision=JD_PREC_BF16,
                 scorer=JD_SCORER_MLP, head_act=JD_ACT_RELU, device=0):
        L = lib()
        cfg = jd_model_config(int(max_tokens), int(max_rows), int(max_markers), precision, scorer, head_act)
        h = C.c_void_p()
        _check(L.jd_model_create(C.byref(cfg), str(weights_path).encode(), int(device), C.byref(h)))
        self.h = h
        self.cfg = cfg

    @classmethod
    def shared(cls, base, max_tokens, max_rows, max_markers, scorer=JD_SCORER_MLP, head_act=JD_ACT_RELU):
        """jd_model_create_shared: a handle on base's weights with its own workspace
        (for another stream / host thread); keeps base alive."""
        self = cls.__new__(cls)
        cfg = jd_model_config(int(max_tokens), int(max_rows), int(max_markers), base.cfg.precision, scorer, head_act)
        h = C.c_void_p()
        _check(lib().jd_model_create_shared(base.h, C.byref(cfg), C.byref(h)))
        self.h = h
        self.cfg = cfg
        self.base = base
        return self

    def close(self):
        if getattr(self, "h", None):
            lib().jd_model_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def device_bytes(self):
        return lib().jd_model_device_bytes(self.h)

    @staticmethod
    def device_batch(n_rows, n_tokens, n_markers, max_row_len, tokens, cu_seqlens, mask_pos, opt_off, row_type):
        return jd_batch(n_rows, n_tokens, n_markers, max_row_len, _ptr(tokens), _ptr(cu_seqlens), _ptr(mask_pos),
                        _ptr(opt_off), _ptr(row_type), None, None)

    def jd_decide(self, batch: jd_batch, logits, probs, choice, score, noul, max_p, taps=None, stream=None):
        out = jd_outputs(_ptr(logits), _ptr(probs), _ptr(choice), _ptr(score), _ptr(noul), _ptr(max_p))
        tp = None
        if taps is not None:
            tp = C.byref(jd_taps(_ptr(taps.get("encoder_out")), _ptr(taps.get("marker_state"))))
        _check(lib().jd_decide(self.h, C.byref(batch), C.byref(out), tp, _stream(stream)))

    def jd_forward(self, batch: jd_batch, logits, stream=None):
        _check(lib().jd_forward(self.h, C.byref(batch), _ptr(logits), _stream(stream)))

    def jd_route_host(self, requests, opts: jd_encode_opts, max_tokens=None, max_rows=None, max_markers=None,
                      stream=None):
        """Route requests (objects with state/question/labels); returns dict of
        winner, winner_p, final_candidates [n, 20], final_probs [n, 20], rows_per_round."""
        arr, keep, o, s = _route_marshal(requests)
        c = self.cfg
        _check(lib().jd_route_host(self.h, arr, len(requests), C.byref(opts), int(max_tokens or c.max_tokens),
                                   int(max_rows or c.max_rows), int(max_markers or c.max_markers), C.byref(s),
                                   _stream(stream)))
        return _route_result(o, s)

    def jd_route_device(self, requests, opts: jd_encode_opts, stream=None):
        """jd_route_host with the rounds on the device; the same dict."""
        arr, keep, o, s = _route_marshal(requests)
        _check(lib().jd_route_device(self.h, arr, len(requests), C.byref(opts), C.byref(s), _stream(stream)))
        return _route_result(o, s)

    def jd_forward_noalloc(self, batch: jd_batch, logits, stream=None):
        """jd_forward with every intermediate in the library's static device
        array (no allocation); at most 1024 tokens, 32 rows, 128 markers."""
        _check(lib().jd_forward_noalloc(self.h, C.byref(batch), _ptr(logits), _stream(stream)))

    def jd_noalloc_check_status(self, stream=None):
        """Synchronize `stream` and raise JDError if the last jd_forward_noalloc
        call's kernels recorded a failed check."""
        _check(lib().jd_noalloc_check_status(self.h, _stream(stream)))

    def jd_check_status(self):
        _check(lib().jd_check_status(self.h))

    def jd_set_graph_mode(self, enable):
        _check(lib().jd_set_graph_mode(self.h, int(bool(enable))))

    def jd_graph_stats(self):
        """(graphs captured, calls served by replaying an earlier capture, buckets held)."""
        c, r, b = C.c_int64(), C.c_int64(), C.c_int32()
        _check(lib().jd_graph_stats(self.h, C.byref(c), C.byref(r), C.byref(b)))
        return c.value, r.value, b.value

    def jd_last_launch_count(self):
        return lib().jd_last_launch_count(self.h)

    def jd_set_profiling(self, enable):
        _check(lib().jd_set_profiling(self.h, int(bool(enable))))

    def jd_profile_report(self):
        """{kernel name: (launches, total ms)} summed since profiling was enabled."""
        buf = C.create_string_buffer(1 << 16)
        _check(lib().jd_profile_report(self.h, buf, len(buf)))
        out = {}
        for line in buf.value.decode().splitlines():
            name, n, ms = line.split()
            out[name] = (int(n), float(ms))
        return out

    def _host_out(self, n_rows, n_markers):
        o = dict(logits=np.zeros(n_markers, np.float32), probs=np.zeros(n_markers, np.float32),
                 choice=np.zeros(n_rows, np.int32), score=np.zeros(n_rows, np.float32),
                 noul=np.zeros(n_rows, np.float32), max_p=np.zeros(n_rows, np.float32))
        s = jd_host_outputs(o["logits"].ctypes.data_as(f32p), o["probs"].ctypes.data_as(f32p),
                            o["choice"].ctypes.data_as(i32p), o["score"].ctypes.data_as(f32p),
                            o["noul"].ctypes.data_as(f32p), o["max_p"].ctypes.data_as(f32p), 0, 0)
        return o, s

    def jd_decide_host(self, rows, opts: jd_encode_opts, stream=None):
        keep = _RowKeep(rows)
        n_m = sum(len(r.options) for r in rows)
        o, s = self._host_out(len(rows), n_m)
        _check(lib().jd_decide_host(self.h, keep.arr, len(rows), C.byref(opts), C.byref(s), _stream(stream)))
        return o

    def jd_decide_host_submit(self, rows, opts: jd_encode_opts, stream=None):
        """Queue one host batch (at most two in flight); returns its ticket."""
        keep = _RowKeep(rows)
        t = C.c_int64()
        _check(lib().jd_decide_host_submit(self.h, keep.arr, len(rows), C.byref(opts), _stream(stream), C.byref(t)))
        self._inflight = getattr(self, "_inflight", {})
        self._inflight[t.value] = (len(rows), sum(len(r.options) for r in rows))
        return t.value

    def jd_decide_host_collect(self, ticket):
        """Outputs of the oldest call in flight (the dict of jd_decide_host)."""
        n_rows, n_m = self._inflight.pop(ticket)
        o, s = self._host_out(n_rows, n_m)
        _check(lib().jd_decide_host_collect(self.h, ticket, C.byref(s)))
        return o

    def jd_decide_packed_host(self, hb: HostBatch, stream=None):
        o, s = self._host_out(hb.n_rows, hb.n_markers)
        bs = hb.as_struct()
        _check(lib().jd_decide_packed_host(self.h, C.byref(bs), C.byref(s), _stream(stream)))
        return o
