"""ctypes loader for libkld.so: prototypes of the C ABI in include/kld.h.

Loading needs no GPU (the CUDA runtime is linked statically); calls that
launch kernels need one.  A missing library is an error, never a fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkld.so")

KLD_OK = 0
KLD_ERR_INVALID_ARG = 1
KLD_ERR_ALIGNMENT = 2
KLD_ERR_UNSUPPORTED = 3
KLD_ERR_WORKSPACE = 4
KLD_ERR_CUDA = 5

KLD_DEV_BAD_TARGET = 0x1
KLD_DEV_BAD_ID = 0x2
KLD_DEV_TIMEOUT = 0x4

KLD_F32 = 0
KLD_BF16 = 1

KLD_NOALLOC_MAX_ROWS = 32768

KLD_MAX_QUANTILES = 8
KLD_MAX_THRESHOLDS = 8


class KldStats(ctypes.Structure):
    """Mirror of struct kld_stats (include/kld.h)."""
    _fields_ = [
        ("n", ctypes.c_int64),
        ("n_nan", ctypes.c_int64),
        ("top1_agree", ctypes.c_int64),
        ("exceed", ctypes.c_int64 * KLD_MAX_THRESHOLDS),
        ("mean_kl", ctypes.c_double),
        ("top1_rate", ctypes.c_double),
        ("ref_mean_nll", ctypes.c_double),
        ("cand_mean_nll", ctypes.c_double),
        ("ref_ppl", ctypes.c_double),
        ("cand_ppl", ctypes.c_double),
        ("ppl_ratio", ctypes.c_double),
        ("q_value", ctypes.c_double * KLD_MAX_QUANTILES),
        ("q_lo", ctypes.c_float * KLD_MAX_QUANTILES),
        ("q_hi", ctypes.c_float * KLD_MAX_QUANTILES),
        ("nq", ctypes.c_int32),
        ("nt", ctypes.c_int32),
    ]


assert ctypes.sizeof(KldStats) == 280

class KldPaired(ctypes.Structure):
    """Mirror of struct kld_paired (include/kld.h)."""
    _fields_ = [
        ("n_ctx", ctypes.c_int64),
        ("n_pos", ctypes.c_int64),
        ("a_lower", ctypes.c_int64),
        ("b_lower", ctypes.c_int64),
        ("ties", ctypes.c_int64),
        ("n_boot", ctypes.c_int64),
        ("mean_a", ctypes.c_double),
        ("mean_b", ctypes.c_double),
        ("diff", ctypes.c_double),
        ("ci", ctypes.c_double * KLD_MAX_QUANTILES),
        ("nq", ctypes.c_int32),
        ("pad", ctypes.c_int32),
    ]


assert ctypes.sizeof(KldPaired) == 144

KLD_SPARSE_MAX_K = 1024
KLD_CAPTURE_CANDIDATES = 8192
KLD_SHARD_STEPS = 5

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); every symbol declared in include/kld.h
PROTOTYPES = {
    "kld_version": (ctypes.c_int, []),
    "kld_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kld_full_vocab": (ctypes.c_int, [_P, _P, ctypes.c_int, _I64, _I64, _I64, _I64, _P, _P, _P, _P,
                                      _P, _P, _P, _SZ, _P, _P]),
    "kld_full_vocab_workspace_size": (_SZ, [_I64]),
    "kld_full_vocab_noalloc": (ctypes.c_int, [_P, _P, ctypes.c_int, _I64, _I64, _I64, _I64, _P, _P, _P,
                                              _P, _P, _P, _P, _P]),
    "kld_topk_tail": (ctypes.c_int, [_P, _P, _P, _P, _I64, _I32, _I64, _P, _P, _P, _P, _P]),
    "kld_sparse_ref_workspace_size": (_SZ, [_I64, _I32]),
    "kld_sparse_ref_score": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _I32, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _SZ, _P, _P]),
    "kld_sparse_capture_workspace_size": (_SZ, [_I64, _I32]),
    "kld_sparse_capture": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _SZ, _P, _P]),
    "kld_shared_head_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "kld_from_hidden_shared_head": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P,
                                                   _SZ, _P, _P]),
    "kld_reduce_workspace_size": (_SZ, [_I64]),
    "kld_reduce_shard_block_bytes": (_SZ, []),
    "kld_reduce_shard_workspace_size": (_SZ, [_I64]),
    "kld_reduce_shard_step": (ctypes.c_int, [_I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I32, _P, _I32,
                                             _P, _P, _SZ, _P, _P]),
    "kld_reduce_stats": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I64, _P, _I32, _P, _I32, _P, _P,
                                        _SZ, _P, _P]),
    "kld_paired_workspace_size": (_SZ, [_I64, _I32, _I32]),
    "kld_paired_compare": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _P, _I32, _P, _I32, _P, _I32, _P, _P, _P, _SZ,
                                          _P, _P]),
}

# exported for tests only (not part of the public header)
TEST_PROTOTYPES = {
    "kld_sparse_capture_exact": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _SZ,
                                                _P, _P]),
    "kld_sparse_ref_score_split": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, _I64, _P, _I32, _P, _P, _P, _P,
                                                  _P, _P, _P, _P, _SZ, _P, _P, _I32]),
    "kld_from_hidden_shared_head_withhold": (ctypes.c_int, [_P, _P, _P, _I64, _I64, _I64, _P, _P, _SZ, _P, _P]),
    "kld_reduce_stats_withhold": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I64, _P, _I32, _P, _I32, _P, _P,
                                                 _SZ, _P, _P]),
    "kld_full_vocab_split": (ctypes.c_int, [_P, _P, ctypes.c_int, _I64, _I64, _I64, _I64, _P, _P, _P,
                                            _P, _P, _P, _P, _SZ, _P, _P, _I32]),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkld.so not found at {LIB_PATH}; build it with "
            "`python -m quantization_fidelity_scoring_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for table in (PROTOTYPES, TEST_PROTOTYPES):
        for name, (res, args) in table.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
    _lib = lib
    return lib
