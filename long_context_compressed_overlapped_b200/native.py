"""ctypes mirror of include/csahca.h and the loader of libcsahca.so.

Argument marshalling only.  Loading fails loudly if the library is missing:
there is no other implementation to fall back to.
"""

from __future__ import annotations

import ctypes as C
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libcsahca.so")

ABI_VERSION = 4                     # CSAHCA_ABI_VERSION of the mirrored header

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_ALIGNMENT = -3
ERR_WORKSPACE = -4
ERR_LAUNCH = -5
ERR_DEVICE_TIMEOUT = -6
ERR_NO_DEVICE = -7

NOALLOC_SCRATCH_BYTES = 32 << 20    # CSAHCA_NOALLOC_SCRATCH_BYTES
CP_MAX_RANKS = 64                   # CSAHCA_CP_MAX_RANKS

F32, BF16, E4M3 = 0, 1, 2
CSA, HCA = 0, 1

i32, f32, vp, sz = C.c_int32, C.c_float, C.c_void_p, C.c_size_t


class CompressArgs(C.Structure):
    _fields_ = [("dtype", i32), ("B", i32), ("n", i32), ("c", i32), ("m", i32),
                ("first_block", i32), ("num_blocks", i32), ("rms_norm", i32),
                ("rope_dims", i32), ("rope_base", f32), ("eps", f32), ("reserved0", i32),
                ("a", vp), ("b", vp), ("za", vp), ("zb", vp), ("bias_a", vp), ("bias_b", vp),
                ("gain", vp), ("out", vp)]


class IndexerArgs(C.Structure):
    _fields_ = [("q_dtype", i32), ("k_dtype", i32), ("B", i32), ("nq", i32), ("HI", i32),
                ("dI", i32), ("N", i32), ("m", i32), ("k", i32), ("entry_base", i32),
                ("qI", vp), ("w", vp), ("kI", vp), ("kI_scale", vp), ("q_pos", vp),
                ("idx", vp), ("scores_out", vp), ("sel_scores", vp), ("workspace", vp),
                ("workspace_bytes", sz)]


class AttnArgs(C.Structure):
    _fields_ = [("kind", i32), ("dtype", i32), ("B", i32), ("n", i32), ("H", i32), ("d", i32),
                ("N", i32), ("m", i32), ("k", i32), ("w", i32), ("rope_dims", i32),
                ("rope_base", f32), ("eps", f32), ("scale", f32), ("q_norm", i32),
                ("kv_norm", i32),
                ("q", vp), ("kv_comp", vp), ("kv_win", vp), ("q_gain", vp), ("kv_gain", vp),
                ("idx", vp), ("sinks", vp), ("out", vp), ("workspace", vp),
                ("workspace_bytes", sz)]


class DecodeArgs(C.Structure):
    _fields_ = [("kind", i32), ("dtype", i32), ("B", i32), ("H", i32), ("d", i32),
                ("N_cap", i32), ("m", i32), ("w", i32), ("rope_dims", i32), ("rope_base", f32),
                ("eps", f32), ("scale", f32), ("q_norm", i32), ("k", i32), ("HI", i32),
                ("dI", i32), ("qI_dtype", i32), ("kI_dtype", i32), ("kv_dtype", i32),
                ("entry_base", i32), ("q", vp), ("pos", vp), ("q_gain", vp), ("kv_cache", vp),
                ("win", vp), ("sinks", vp), ("qI", vp), ("wI", vp), ("kI", vp), ("kI_scale", vp),
                ("idx_in", vp), ("idx_out", vp), ("out", vp), ("partial_out", vp),
                ("skip_window", i32), ("reserved2", i32), ("workspace", vp), ("workspace_bytes", sz)]


class DecodeCompressArgs(C.Structure):
    _fields_ = [("kind", i32), ("dtype", i32), ("B", i32), ("d", i32), ("m", i32),
                ("N_cap", i32), ("w", i32), ("rope_dims", i32), ("rope_base", f32), ("eps", f32),
                ("kv_norm", i32), ("dI", i32), ("kI_dtype", i32), ("kv_dtype", i32),
                ("entry_base", i32), ("reserved1", i32), ("pos", vp), ("kv_raw", vp), ("a", vp), ("b", vp), ("za", vp), ("zb", vp),
                ("bias_a", vp), ("bias_b", vp), ("kv_gain", vp), ("ring", vp), ("kv_cache", vp),
                ("win", vp), ("ia", vp), ("ib", vp), ("iza", vp), ("izb", vp), ("ibias_a", vp),
                ("ibias_b", vp), ("iring", vp), ("kI", vp), ("kI_scale", vp)]


class CpTopkMergeArgs(C.Structure):
    _fields_ = [("R", i32), ("rows", i32), ("k", i32), ("rank", i32), ("bases", vp),
                ("cand_idx", vp), ("cand_scores", vp), ("idx_global", vp), ("idx_local", vp)]


class CpMergeArgs(C.Structure):
    _fields_ = [("dtype", i32), ("R", i32), ("rows", i32), ("H", i32), ("d", i32),
                ("rope_dims", i32), ("rope_base", f32), ("reserved0", i32),
                ("partials", vp), ("sinks", vp), ("pos", vp), ("out", vp)]


class TraceEntry(C.Structure):
    _fields_ = [("name", C.c_char * 48), ("launches", C.c_int64), ("total_ms", C.c_double)]


STRUCTS = {0: CompressArgs, 1: IndexerArgs, 2: AttnArgs, 3: DecodeArgs, 4: DecodeCompressArgs,
           5: CpTopkMergeArgs, 6: CpMergeArgs}

# Every symbol include/csahca.h declares, with (restype, argtypes).
SIGNATURES = {
    "csa_compress": (C.c_int, [C.POINTER(CompressArgs), vp]),
    "hca_compress": (C.c_int, [C.POINTER(CompressArgs), vp]),
    "indexer_topk": (C.c_int, [C.POINTER(IndexerArgs), vp]),
    "csahca_indexer_workspace_size": (sz, [C.POINTER(IndexerArgs)]),
    "indexer_topk_noalloc": (C.c_int, [C.POINTER(IndexerArgs), vp]),
    "compressed_attn_prefill": (C.c_int, [C.POINTER(AttnArgs), vp]),
    "csahca_prefill_workspace_size": (sz, [C.POINTER(AttnArgs)]),
    "compressed_attn_decode": (C.c_int, [C.POINTER(DecodeArgs), vp]),
    "csahca_decode_workspace_size": (sz, [C.POINTER(DecodeArgs)]),
    "decode_compress": (C.c_int, [C.POINTER(DecodeCompressArgs), vp]),
    "cp_topk_merge": (C.c_int, [C.POINTER(CpTopkMergeArgs), vp]),
    "cp_attn_merge": (C.c_int, [C.POINTER(CpMergeArgs), vp]),
    "csahca_status_string": (C.c_char_p, [C.c_int]),
    "csahca_abi_version": (C.c_int, []),
    "csahca_kv_row_bytes": (C.c_int64, [C.c_int32, C.c_int32, C.c_int32]),
    "csahca_struct_size": (C.c_int64, [C.c_int]),
    "csahca_device_error": (C.c_int, [vp, C.POINTER(i32)]),
    "csahca_selftest_bounded_wait": (C.c_int, [vp]),
    "csahca_trace_enable": (C.c_int, [C.c_int]),
    "csahca_trace_collect": (C.c_int, [C.POINTER(TraceEntry), C.c_int, C.POINTER(C.c_int)]),
}

_lib = None


class CsahcaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().csahca_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {msg} (status {status})")


def lib():
    """Load libcsahca.so (once) and check that the ctypes struct mirrors
    have the library's sizes."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m long_context_compressed_overlapped_b200.build`")
    h = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(h, name)
        fn.restype = res
        fn.argtypes = args
    if h.csahca_abi_version() != ABI_VERSION:
        raise RuntimeError(f"ABI mismatch: library version {h.csahca_abi_version()}, binding {ABI_VERSION}")
    for which, st in STRUCTS.items():
        got = h.csahca_struct_size(which)
        if got != C.sizeof(st):
            raise RuntimeError(f"ABI mismatch for struct {st.__name__}: library {got}, "
                               f"binding {C.sizeof(st)}")
    _lib = h
    return h


def check(status: int, where: str) -> None:
    if status != OK:
        raise CsahcaError(status, where)
