"""ctypes declarations of libsfc (the C ABI in include/sfc.h).

Argument marshalling only. The library is loaded from this package's
directory; if it is missing the import fails with an error that says how to
build it. There is no fallback implementation.
"""

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# SFC_LIB selects another build of the same library (e.g. a debug build).
LIB_PATH = os.environ.get("SFC_LIB") or os.path.join(_HERE, "libsfc.so")

SFC_NUM_PROTOCOLS = 10
SFC_MAX_RANKS = 8


class Config(C.Structure):
    _fields_ = [("ctas_per_rank", C.c_int), ("timeout_us", C.c_uint32), ("debug_checks", C.c_int),
                ("protocol_mask", C.c_uint32), ("device_epochs", C.c_int)]


SFC_COST_BUCKETS = 24
SFC_COST_MIN_LOG2 = 9


class CostEntry(C.Structure):
    _fields_ = [("alpha_us", C.c_double), ("beta_us_per_byte", C.c_double),
                ("table_us", C.c_double * SFC_COST_BUCKETS)]


class CostModel(C.Structure):
    _fields_ = [("c", CostEntry * (SFC_MAX_RANKS + 1) * SFC_NUM_PROTOCOLS * 2)]


class LLView(C.Structure):
    _fields_ = [("scratch", C.c_void_p), ("slot_stride", C.c_uint64), ("nranks", C.c_int),
                ("status", C.c_void_p), ("timeout_ns", C.c_uint64)]


SFC_FLOOR_SMS = 8
SFC_FLOOR_LOCATIONS = 8


class FloorResult(C.Structure):
    _fields_ = [("flag_rtt_ns_p50", C.c_double), ("flag_rtt_ns_p10", C.c_double), ("flag_rtt_ns_p90", C.c_double),
                ("flag_rtt_ns_min_pair", C.c_double), ("flag_rtt_ns_max_pair", C.c_double),
                ("flag_rtt_ns_by_location", C.c_double * SFC_FLOOR_LOCATIONS),
                ("initiator_sm", C.c_int * SFC_FLOOR_SMS), ("responder_sm", C.c_int * SFC_FLOOR_SMS),
                ("pairs", C.c_int), ("l2_rtt_ns_p50", C.c_double), ("sm_clock_ghz", C.c_double),
                ("globaltimer_step_ns", C.c_double)]


# (name, restype, argtypes) for every entry point of include/sfc.h
_P = C.c_void_p
_S = C.c_int
SIGNATURES = [
    ("sfc_init", _S, [C.POINTER(_P), C.c_int, C.c_size_t, C.POINTER(Config)]),
    ("sfc_destroy", _S, [_P]),
    ("sfc_reset", _S, [_P, _P]),
    ("sfc_allreduce", _S, [_P, C.POINTER(_P), C.POINTER(_P), C.c_size_t, C.c_int, C.c_int, C.c_uint32, _P]),
    ("sfc_allgather", _S, [_P, C.POINTER(_P), C.POINTER(_P), C.c_size_t, C.c_int, C.c_int, C.c_uint32, _P]),
    ("sfc_allreduce_chain", _S, [_P, C.c_int, _P, _P, C.c_size_t, C.c_int, C.c_int, C.c_uint32, _P, _P, _P]),
    ("sfc_allgather_chain", _S, [_P, C.c_int, _P, _P, C.c_size_t, C.c_int, C.c_int, C.c_uint32, _P, _P, _P]),
    ("sfc_allreduce_chain_host", _S, [_P, C.c_int, _P, _P, C.c_size_t, C.c_int, C.c_int, C.c_uint32, _P, _P]),
    ("sfc_select_protocol", C.c_int, [_P, C.c_int, C.c_size_t, C.c_int]),
    ("sfc_select_protocol_model", C.c_int, [C.POINTER(CostModel), C.c_int, C.c_size_t, C.c_int]),
    ("sfc_set_cost_model", _S, [_P, C.POINTER(CostModel)]),
    ("sfc_cost_estimate", C.c_double, [C.POINTER(CostModel), C.c_int, C.c_int, C.c_size_t, C.c_int]),
    ("sfc_default_cost_model", None, [C.POINTER(CostModel)]),
    ("sfc_algorithmic_bytes", C.c_double, [C.c_int, C.c_int, C.c_size_t, C.c_int]),
    ("sfc_get_status", _S, [_P, C.POINTER(C.c_uint32)]),
    ("sfc_status_string", C.c_char_p, [C.c_int]),
    ("sfc_next_epoch", C.c_uint32, [_P]),
    ("sfc_launch_shape", _S, [_P, C.c_int, C.c_int, C.c_size_t, C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    ("sfc_scratch_slot", _S, [_P, C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(_P), C.POINTER(C.c_size_t)]),
    ("sfc_set_silent_rank", _S, [_P, C.c_int]),
    ("sfc_measure_floor", _S, [C.c_int, C.POINTER(FloorResult)]),
    ("sfc_launch_count", C.c_uint64, [_P]),
    ("sfc_check_guards", _S, [_P]),
    ("sfc_get_ll_view", _S, [_P, C.POINTER(LLView)]),
    ("sfc_reserve_epochs", _S, [_P, C.c_uint32, C.POINTER(C.c_uint32)]),
    ("sfc_linear_allreduce", _S, [_P, C.POINTER(_P), C.POINTER(_P), C.POINTER(_P), C.c_size_t, C.c_size_t,
                                  C.c_uint32, _P]),
    ("sfc_linear_allreduce_tokens", _S, [_P, C.POINTER(_P), C.POINTER(_P), C.POINTER(_P), C.c_size_t, C.c_size_t,
                                          C.c_uint32, C.c_uint32, _P]),
    ("sfc_plan_create", _S, [_P, C.c_int, C.POINTER(_P), C.POINTER(_P), C.c_size_t, C.c_int, C.c_int,
                             C.POINTER(_P)]),
    ("sfc_plan_launch", _S, [_P, _P]),
    ("sfc_plan_destroy", _S, [_P]),
    ("sfc_allreduce_noalloc", _S, [C.POINTER(_P), C.POINTER(_P), C.c_int, C.c_size_t, _P]),
    ("sfc_noalloc_status", _S, [_P, C.POINTER(C.c_uint32)]),
]

_lib = None


def load():
    """The loaded library (ctypes.CDLL) with every signature declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m latency_self_synchronizing_b200.build` "
            "(the CUDA library is required; there is no fallback)")
    lib = C.CDLL(LIB_PATH)
    for name, res, args in SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
