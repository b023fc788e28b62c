"""B200 (sm_100a) library for the Julia-1 decision-model forward pass.

The compute path lives in libjulia_decide.so (hand-written CUDA for sm_100a,
C ABI in include/julia_decide.h); this package only builds and binds it.
"""
from ._lib import (  # noqa: F401
    JDError, Model, HostBatch, jd_serialize, jd_version, encode_opts, lib,
    JD_OK, JD_ERR_INVALID_ARG, JD_ERR_OPTION_COUNT, JD_ERR_OVERFLOW, JD_ERR_TOKEN_RANGE, JD_ERR_CAPACITY,
    JD_ERR_CUDA, JD_ERR_DEVICE_STATUS, JD_ERR_IO, JD_PREC_BF16, JD_PREC_FP32, JD_SCORER_MLP, JD_SCORER_LINEAR,
    JD_ACT_RELU, JD_ACT_GELU,
)
