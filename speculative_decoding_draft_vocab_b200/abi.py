"""ctypes binding of ``include/dspark.h``: the same entry points, argument marshalling only.

Loading this module loads ``libdspark.so`` from the package directory and raises if it
is missing: there is no fallback path of any kind.  Every step of the loss runs in
the library's CUDA kernels; PyTorch only supplies device memory and the stream.
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdspark.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libdspark.so is not built ({LIB_PATH}); run "
        "`python -m speculative_decoding_draft_vocab_b200.build` first")
lib = ctypes.CDLL(LIB_PATH)

c_i64 = ctypes.c_int64
c_vp = ctypes.c_void_p

# status codes
DSPARK_OK = 0
DSPARK_ERR_INVALID_ARG = 1
DSPARK_ERR_MISSING_TARGET = 2
DSPARK_ERR_ID_OUT_OF_RANGE = 3
DSPARK_ERR_ALIGNMENT = 4
DSPARK_ERR_WORKSPACE = 5
DSPARK_ERR_UNSUPPORTED = 6
DSPARK_ERR_DEVICE_TIMEOUT = 7
DSPARK_ERR_CUDA = 8

DSPARK_F32 = 0
DSPARK_BF16 = 1

REPORT_KEYS = ("loss", "ce", "l1", "conf", "accept", "tau")  # DSPARK_REP_* order
DSPARK_REP_COUNT = len(REPORT_KEYS)


class dspark_problem_t(ctypes.Structure):
    _fields_ = [
        ("B", c_i64), ("N", c_i64), ("K", c_i64), ("V", c_i64),
        ("logits_dtype", c_i64),
        ("draft_logits", c_vp), ("draft_ld", c_i64),
        ("target_logits", c_vp), ("target_ld", c_i64),
        ("target_ids", c_vp),
        ("eval_mask", c_vp),
        ("block_keep", c_vp),
        ("confidence_logits", c_vp),
        ("target_hidden", c_vp), ("lm_head", c_vp), ("target_hidden_size", c_i64),
        ("prev_ids", c_vp), ("valid", c_vp), ("target_vocab", c_i64),
        ("markov_w1", c_vp), ("markov_w2", c_vp), ("markov_rank", c_i64),
        ("draft_hidden", c_vp), ("hidden_size", c_i64),
        ("conf_w", c_vp), ("conf_b", c_vp), ("conf_with_markov", c_i64),
        ("target_norm_weight", c_vp), ("target_norm_eps", ctypes.c_float),
    ]


class dspark_params_t(ctypes.Structure):
    _fields_ = [
        ("ce_alpha", ctypes.c_float), ("l1_alpha", ctypes.c_float),
        ("conf_alpha", ctypes.c_float), ("gamma", ctypes.c_float),
        ("gamma_enabled", ctypes.c_int32), ("invalid_row_mode", ctypes.c_int32),
    ]


class dspark_fwd_out_t(ctypes.Structure):
    _fields_ = [
        ("loss_num", c_vp), ("num_tokens", c_vp), ("report", c_vp),
        ("ce_rows", c_vp), ("l1_rows", c_vp), ("accept_rows", c_vp), ("conf_rows", c_vp),
    ]


class dspark_grads_t(ctypes.Structure):
    _fields_ = [
        ("grad_scale", c_vp),
        ("dlogits", c_vp), ("dlogits_ld", c_i64),
        ("dconf", c_vp),
        ("dW1", c_vp), ("dW2", c_vp), ("dconf_w", c_vp), ("dconf_b", c_vp),
        ("dhidden", c_vp),
        ("accumulate", c_i64),
    ]


class dspark_tp_t(ctypes.Structure):
    _fields_ = [("tp_size", c_i64), ("vocab_begin", c_i64), ("vocab_size", c_i64)]


# floats per row of the two exchange records of the vocabulary-parallel path
DSPARK_TP_REC1_FLOATS = 8
DSPARK_TP_REC2_FLOATS = 4

P = ctypes.POINTER
lib.dspark_workspace_size.argtypes = [P(dspark_problem_t)]
lib.dspark_workspace_size.restype = ctypes.c_size_t
lib.dspark_loss_fwd.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_fwd_out_t),
                                P(dspark_grads_t), c_vp, ctypes.c_size_t, c_vp]
lib.dspark_loss_fwd.restype = ctypes.c_int
lib.dspark_loss_bwd.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_grads_t),
                                c_vp, ctypes.c_size_t, c_vp]
lib.dspark_loss_bwd.restype = ctypes.c_int
lib.dspark_loss_fwd_noalloc.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_fwd_out_t),
                                        P(dspark_grads_t), c_vp]
lib.dspark_loss_fwd_noalloc.restype = ctypes.c_int
lib.dspark_acceptance.argtypes = [c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]
lib.dspark_acceptance.restype = ctypes.c_int
lib.dspark_tp_partials.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_tp_t), c_vp, c_vp,
                                   ctypes.c_size_t, c_vp]
lib.dspark_tp_partials.restype = ctypes.c_int
lib.dspark_tp_l1.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_tp_t), c_vp, c_vp, c_vp,
                             ctypes.c_size_t, c_vp]
lib.dspark_tp_l1.restype = ctypes.c_int
lib.dspark_tp_finish.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_tp_t), c_vp,
                                 P(dspark_fwd_out_t), P(dspark_grads_t), c_vp, c_vp, ctypes.c_size_t, c_vp]
lib.dspark_tp_finish.restype = ctypes.c_int
lib.dspark_tp_heads_bwd.argtypes = [P(dspark_problem_t), P(dspark_params_t), P(dspark_tp_t), c_vp,
                                    P(dspark_grads_t), c_vp, ctypes.c_size_t, c_vp]
lib.dspark_tp_heads_bwd.restype = ctypes.c_int
lib.dspark_check_status.argtypes = [c_vp, c_vp]
lib.dspark_check_status.restype = ctypes.c_int
lib.dspark_status_string.argtypes = [ctypes.c_int]
lib.dspark_status_string.restype = ctypes.c_char_p
lib.dspark_last_cuda_error.argtypes = []
lib.dspark_last_cuda_error.restype = ctypes.c_char_p

# The C entry points under their own names.
dspark_workspace_size = lib.dspark_workspace_size
dspark_loss_fwd = lib.dspark_loss_fwd
dspark_loss_bwd = lib.dspark_loss_bwd
dspark_loss_fwd_noalloc = lib.dspark_loss_fwd_noalloc
# The fixed scratch of dspark_loss_fwd_noalloc: the rows (B*N*K) and the workspace bytes
# it serves (DSPARK_NOALLOC_MAX_ROWS, DSPARK_NOALLOC_BYTES of dspark.h).
NOALLOC_MAX_ROWS = 8192
NOALLOC_BYTES = 467200
dspark_acceptance = lib.dspark_acceptance
dspark_tp_partials = lib.dspark_tp_partials
dspark_tp_l1 = lib.dspark_tp_l1
dspark_tp_finish = lib.dspark_tp_finish
dspark_tp_heads_bwd = lib.dspark_tp_heads_bwd
dspark_check_status = lib.dspark_check_status
dspark_status_string = lib.dspark_status_string
dspark_last_cuda_error = lib.dspark_last_cuda_error


class DSparkError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = f", {dspark_last_cuda_error().decode()}" if status == DSPARK_ERR_CUDA else ""
        super().__init__(f"{where}: {dspark_status_string(status).decode()} (status {status}{detail})")


def check(status: int, where: str) -> None:
    if status != DSPARK_OK:
        raise DSparkError(status, where)
