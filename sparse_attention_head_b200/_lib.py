"""ctypes loader for libea.so (the C ABI declared in include/ea.h).

The library is built in-tree by ``sparse_attention_head_b200.build``.  There
is no fallback: if the library is missing or fails to load, every entry point
raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libea.so")

EA_OK = 0
EA_ERR_INVALID_ARG = 1
EA_ERR_UNSUPPORTED = 2
EA_ERR_MISALIGNED = 3
EA_ERR_CUDA = 4
EA_ERR_TIMEOUT = 5
EA_ERR_WORKSPACE = 6
EA_ERR_SCRATCH_LIMIT = 7

# bytes of the fixed device scratch behind ea_router_decide_noalloc
EA_ROUTER_NOALLOC_MAX_BYTES = 1 << 20

EA_SELECT_ALL = 0
EA_SELECT_FA = 1
EA_SELECT_SA = 2

EXPORTED = [
    "ea_status_string", "ea_version",
    "ea_router_workspace_size", "ea_router_decide", "ea_router_decide_noalloc",
    "ea_hybrid_attn_workspace_size", "ea_hybrid_attn_prefill",
    "ea_get_device_status", "ea_schedule_units", "ea_schedule_unit_tiles",
    "ea_attn_grid_size", "ea_decode_workspace_size", "ea_hybrid_attn_decode",
    "ea_decode_kv_policy", "ea_hybrid_attn_varlen_workspace_size",
    "ea_hybrid_attn_prefill_varlen", "ea_schedule_units_varlen",
    "ea_router_varlen_workspace_size", "ea_router_decide_varlen",
    "ea_hybrid_attn_routed_workspace_size", "ea_hybrid_attn_prefill_routed",
    "ea_hybrid_attn_varlen_routed_workspace_size", "ea_hybrid_attn_prefill_varlen_routed",
    "ea_hybrid_attn_prefill_lse", "ea_hybrid_attn_backward_workspace_size",
    "ea_hybrid_attn_backward", "ea_router_gumbel_workspace_size", "ea_router_decide_gumbel",
    "ea_router_ste_backward_workspace_size", "ea_router_ste_backward",
    "ea_hybrid_attn_prefill_train", "ea_fp8_vt_stride", "ea_quantize_fp8_workspace_size",
    "ea_quantize_fp8", "ea_hybrid_attn_prefill_fp8", "ea_hybrid_attn_host_workspace_size",
    "ea_hybrid_attn_host_chunks", "ea_hybrid_attn_prefill_host", "ea_shutdown",
    "ea_hybrid_attn_prefill_traced", "ea_router_pool_rows", "ea_router_mlp_workspace_size",
    "ea_router_mlp", "ea_hybrid_attn_prefill_groups", "ea_hybrid_attn_prefill_heads",
]


class EaAttnParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("sink", ctypes.c_int),
                ("window", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("select", ctypes.c_int)]


class EaVarlenParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("total", ctypes.c_int), ("max_seqlen", ctypes.c_int), ("d", ctypes.c_int),
                ("sink", ctypes.c_int), ("window", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("select", ctypes.c_int)]


class EaDecodeParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("sink", ctypes.c_int), ("window", ctypes.c_int),
                ("max_len", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("n_full", ctypes.c_int), ("n_sa", ctypes.c_int)]


class EaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} (status {code})")


_lib = None


def load(build_if_missing: bool = False) -> ctypes.CDLL:
    """Load libea.so once; raise if it is missing (no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        if build_if_missing:
            from . import build
            build.build()
        else:
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_attention_head_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    c_size, c_int, c_float, vp = ctypes.c_size_t, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    pparams = ctypes.POINTER(EaAttnParams)
    lib.ea_status_string.restype = ctypes.c_char_p
    lib.ea_status_string.argtypes = [c_int]
    lib.ea_version.restype = c_int
    lib.ea_version.argtypes = []
    lib.ea_router_workspace_size.restype = c_size
    lib.ea_router_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.ea_router_decide.restype = c_int
    lib.ea_router_decide.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp,
                                     c_int, c_float, vp, vp, vp, c_size, vp]
    lib.ea_router_decide_noalloc.restype = c_int
    lib.ea_router_decide_noalloc.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, c_int, vp,
                                             vp, c_int, c_float, vp, vp, vp]
    lib.ea_hybrid_attn_workspace_size.restype = c_size
    lib.ea_hybrid_attn_workspace_size.argtypes = [pparams]
    lib.ea_hybrid_attn_host_workspace_size.restype = c_size
    lib.ea_hybrid_attn_host_workspace_size.argtypes = [pparams, c_int]
    lib.ea_hybrid_attn_prefill_traced.restype = c_int
    lib.ea_hybrid_attn_prefill_traced.argtypes = [vp, vp, vp, vp, pparams, vp, vp, c_size, vp,
                                                  c_int, vp]
    lib.ea_shutdown.restype = c_int
    lib.ea_shutdown.argtypes = []
    lib.ea_hybrid_attn_host_chunks.restype = c_int
    lib.ea_hybrid_attn_host_chunks.argtypes = [pparams, c_int]
    lib.ea_hybrid_attn_prefill_host.restype = c_int
    lib.ea_hybrid_attn_prefill_host.argtypes = [vp, vp, vp, vp, vp, vp, c_int, vp, vp, c_float,
                                                pparams, vp, vp, c_int, vp, c_size, vp]
    lib.ea_router_pool_rows.restype = c_int
    lib.ea_router_pool_rows.argtypes = [vp, c_int, c_int, c_int, c_int, c_int, c_int, vp, vp,
                                        c_size, vp]
    lib.ea_router_mlp_workspace_size.restype = c_size
    lib.ea_router_mlp_workspace_size.argtypes = [c_int, c_int]
    lib.ea_router_mlp.restype = c_int
    lib.ea_router_mlp.argtypes = [vp, c_int, c_int, vp, vp, c_int, vp, vp, c_int, c_float, vp,
                                  vp, vp, c_size, vp]
    lib.ea_hybrid_attn_prefill_groups.restype = c_int
    lib.ea_hybrid_attn_prefill_groups.argtypes = [vp, vp, vp, vp, vp, pparams, vp, vp, c_size,
                                                  vp]
    lib.ea_hybrid_attn_prefill_heads.restype = c_int
    lib.ea_hybrid_attn_prefill_heads.argtypes = [vp, vp, vp, vp, vp, pparams, vp, vp, c_size,
                                                 vp]
    lib.ea_hybrid_attn_prefill.restype = c_int
    lib.ea_hybrid_attn_prefill.argtypes = [vp, vp, vp, vp, pparams, vp, vp, c_size, vp]
    lib.ea_get_device_status.restype = c_int
    lib.ea_get_device_status.argtypes = [vp, vp, ctypes.POINTER(c_int)]
    lib.ea_schedule_units.restype = c_int
    lib.ea_schedule_units.argtypes = [vp, pparams, vp, c_int]
    lib.ea_schedule_unit_tiles.restype = c_int
    lib.ea_schedule_unit_tiles.argtypes = [vp, pparams, c_int, vp, vp, c_int]
    lib.ea_attn_grid_size.restype = c_int
    lib.ea_attn_grid_size.argtypes = [pparams, c_int]
    lib.ea_router_varlen_workspace_size.restype = c_size
    lib.ea_router_varlen_workspace_size.argtypes = [c_int, c_int, c_int, c_int]
    lib.ea_router_decide_varlen.restype = c_int
    lib.ea_router_decide_varlen.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp,
                                            c_int, vp, vp, c_int, ctypes.c_float, vp, vp, vp,
                                            c_size, vp]
    pvar = ctypes.POINTER(EaVarlenParams)
    lib.ea_hybrid_attn_varlen_workspace_size.restype = c_size
    lib.ea_hybrid_attn_varlen_workspace_size.argtypes = [pvar]
    lib.ea_hybrid_attn_prefill_varlen.restype = c_int
    lib.ea_hybrid_attn_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, pvar, vp, vp, c_size, vp]
    lib.ea_schedule_units_varlen.restype = c_int
    lib.ea_schedule_units_varlen.argtypes = [vp, pvar, vp, vp, c_int]
    lib.ea_hybrid_attn_routed_workspace_size.restype = c_size
    lib.ea_hybrid_attn_routed_workspace_size.argtypes = [pparams, c_int]
    lib.ea_hybrid_attn_prefill_routed.restype = c_int
    lib.ea_hybrid_attn_prefill_routed.argtypes = [vp, vp, vp, vp, vp, c_int, vp, vp,
                                                  ctypes.c_float, vp, vp, pparams, vp, vp,
                                                  c_size, vp]
    lib.ea_hybrid_attn_varlen_routed_workspace_size.restype = c_size
    lib.ea_hybrid_attn_varlen_routed_workspace_size.argtypes = [pvar, c_int]
    lib.ea_hybrid_attn_prefill_varlen_routed.restype = c_int
    lib.ea_hybrid_attn_prefill_varlen_routed.argtypes = [vp, vp, vp, vp, vp, vp, c_int, vp, vp,
                                                         ctypes.c_float, vp, vp, pvar, vp, vp,
                                                         c_size, vp]
    lib.ea_hybrid_attn_prefill_lse.restype = c_int
    lib.ea_hybrid_attn_prefill_lse.argtypes = [vp, vp, vp, vp, pparams, vp, vp, vp, c_size, vp]
    lib.ea_fp8_vt_stride.restype = c_int
    lib.ea_fp8_vt_stride.argtypes = [c_int]
    lib.ea_quantize_fp8_workspace_size.restype = c_size
    lib.ea_quantize_fp8_workspace_size.argtypes = [c_int]
    lib.ea_quantize_fp8.restype = c_int
    lib.ea_quantize_fp8.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, vp, c_size, vp]
    lib.ea_hybrid_attn_prefill_fp8.restype = c_int
    lib.ea_hybrid_attn_prefill_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, pparams, vp, vp, c_size,
                                               vp]
    lib.ea_hybrid_attn_prefill_train.restype = c_int
    lib.ea_hybrid_attn_prefill_train.argtypes = [vp, vp, vp, vp, pparams, vp, vp, vp, vp, c_size,
                                                 vp]
    lib.ea_hybrid_attn_backward_workspace_size.restype = c_size
    lib.ea_hybrid_attn_backward_workspace_size.argtypes = [pparams]
    lib.ea_hybrid_attn_backward.restype = c_int
    lib.ea_hybrid_attn_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, pparams, vp, vp, vp, vp,
                                            c_size, vp]
    for name in ("ea_router_gumbel_workspace_size", "ea_router_ste_backward_workspace_size"):
        getattr(lib, name).restype = c_size
        getattr(lib, name).argtypes = [c_int] * 6
    lib.ea_router_decide_gumbel.restype = c_int
    lib.ea_router_decide_gumbel.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp,
                                            c_int, vp, vp, ctypes.c_float, vp, vp, vp, vp,
                                            c_size, vp]
    lib.ea_router_ste_backward.restype = c_int
    lib.ea_router_ste_backward.argtypes = [vp, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp,
                                           c_int, vp, vp, ctypes.c_float, vp, vp, vp, vp, vp, vp,
                                           vp, vp, vp, vp, vp, vp, c_size, vp]
    pdec = ctypes.POINTER(EaDecodeParams)
    lib.ea_decode_workspace_size.restype = c_size
    lib.ea_decode_workspace_size.argtypes = [pdec]
    lib.ea_hybrid_attn_decode.restype = c_int
    lib.ea_hybrid_attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, pdec, vp, vp,
                                          c_size, vp]
    lib.ea_decode_kv_policy.restype = c_int
    lib.ea_decode_kv_policy.argtypes = [vp, c_int, c_int, c_int, vp, vp, vp]
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().ea_status_string(int(code)).decode()


def check(code: int, what: str) -> None:
    if code != EA_OK:
        raise EaError(code, what)
