"""ctypes loader for liblca_b200.so (the C ABI of include/lca.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any operation in this package.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblca_b200.so")

LCA_OK = 0
LCA_ERR_INVALID_ARG = -1
LCA_ERR_MISALIGNED = -2
LCA_ERR_WORKSPACE = -3
LCA_ERR_UNSUPPORTED = -4
LCA_ERR_CUDA = -5
LCA_ERR_NO_DEVICE = -6
LCA_ERR_DEVICE_TIMEOUT = -7
LCA_ERR_SCRATCH_LIMIT = -8
NOALLOC_MAX_BATCH = 8

OP_MLA_DECODE, OP_CONDENSE, OP_DECODE_ATTN, OP_DECODE, OP_PREFILL = range(5)
# condensation variants: the method, and the two ablations
VARIANT_LCA, VARIANT_POOL_POSITION, VARIANT_SPARSE = range(3)

# every symbol include/lca.h declares
EXPORTS = ("lca_num_groups", "lca_workspace_bytes", "mla_decode_attn", "lca_condense",
           "lca_decode_attn", "lca_decode", "lca_prefill_block", "lca_strerror",
           "lca_device_status", "lca_profile_enable", "lca_profile_collect", "lca_launch_count",
           "lca_decode_noalloc", "lca_condense_append", "lca_decode_stored",
           "lca_selftest_wait_timeout", "lca_decode_shard", "lca_combine_shards", "lca_decode_varlen",
           "lca_decode_stored_varlen", "lca_append_token")
# floats per head in a shard record: o (512) and its base-2 log-sum-exp
SHARD_RECORD_PER_HEAD = 513


class LcaParams(ctypes.Structure):
    _fields_ = [("g", ctypes.c_int), ("w", ctypes.c_int), ("scale", ctypes.c_float),
                ("variant", ctypes.c_int), ("cache_pitch", ctypes.c_int64)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


class LcaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} ({status})")


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m mla_latent_space_lca_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                            ctypes.c_float)
        L.lca_num_groups.restype = I64
        L.lca_num_groups.argtypes = [I64, LcaParams]
        L.lca_workspace_bytes.restype = SZ
        L.lca_workspace_bytes.argtypes = [I, I, I64, I64, LcaParams]
        L.mla_decode_attn.restype = I
        L.mla_decode_attn.argtypes = [P, P, P, I, I64, F, P, P, P, SZ, P]
        L.lca_condense.restype = I
        L.lca_condense.argtypes = [P, P, I, I64, LcaParams, P, P, P, P, SZ, P]
        L.lca_decode_stored_varlen.restype = I
        L.lca_decode_stored_varlen.argtypes = [P, P, I64, P, P, P, I, I64, LcaParams, P, P, P, SZ, P]
        L.lca_decode_varlen.restype = I
        L.lca_decode_varlen.argtypes = [P, P, P, P, P, I, I64, LcaParams, P, P, P, P, SZ, P]
        L.lca_decode_shard.restype = I
        L.lca_decode_shard.argtypes = [P, P, P, I, I64, I64, I64, LcaParams, P, P, P, SZ, P]
        L.lca_combine_shards.restype = I
        L.lca_combine_shards.argtypes = [P, I, I, P, P, P, P]
        L.lca_selftest_wait_timeout.restype = I
        L.lca_selftest_wait_timeout.argtypes = [P]
        L.lca_append_token.restype = I
        L.lca_append_token.argtypes = [P, P, I, I64, I64, P, P, I, I, P, P]
        L.lca_condense_append.restype = I
        L.lca_condense_append.argtypes = [P, P, I, I64, LcaParams, I64, P, I64, P, P, P, SZ, P]
        L.lca_decode_stored.restype = I
        L.lca_decode_stored.argtypes = [P, P, I64, P, P, I, I64, LcaParams, P, P, P, SZ, P]
        L.lca_decode_attn.restype = I
        L.lca_decode_attn.argtypes = [P, P, P, P, I, I64, LcaParams, P, P, P, SZ, P]
        L.lca_decode.restype = I
        L.lca_decode.argtypes = [P, P, P, P, I, I64, LcaParams, P, P, P, P, SZ, P]
        L.lca_decode_noalloc.restype = I
        L.lca_decode_noalloc.argtypes = [P, P, P, P, I, I64, LcaParams, P, P, P, P]
        L.lca_prefill_block.restype = I
        L.lca_prefill_block.argtypes = [P, P, P, I, I64, I64, I64, LcaParams, P, P, P, P, SZ, P]
        L.lca_strerror.restype = ctypes.c_char_p
        L.lca_strerror.argtypes = [I]
        L.lca_device_status.restype = I
        L.lca_device_status.argtypes = [I, ctypes.POINTER(I)]
        L.lca_profile_enable.restype = I
        L.lca_profile_enable.argtypes = [I]
        L.lca_profile_collect.restype = I
        L.lca_profile_collect.argtypes = [ctypes.POINTER(KernelTime), I]
        L.lca_launch_count.restype = I64
        L.lca_launch_count.argtypes = []
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().lca_strerror(status).decode()


def check(status: int, what: str) -> None:
    if status != LCA_OK:
        raise LcaError(status, what)
