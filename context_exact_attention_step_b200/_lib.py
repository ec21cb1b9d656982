"""ctypes view of ``libcp_attn.so`` (declarations mirror include/cp_attn.h).

Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcp_attn.so")

CP_OK, CP_ERR_INVALID_ARG, CP_ERR_UNSUPPORTED, CP_ERR_ALIGNMENT, CP_ERR_WORKSPACE, CP_ERR_CUDA = range(6)
CP_BF16, CP_FP32 = 0, 1
CP_MASK_NONE, CP_MASK_CAUSAL = 0, 1
CP_LAYOUT_CONTIGUOUS, CP_LAYOUT_ZIGZAG, CP_LAYOUT_STRIPED = 0, 1, 2
CP_SEQ_TO_HEAD, CP_HEAD_TO_SEQ = 0, 1
CP_MAX_CHUNKS = 4
CP_BWD_DQ, CP_BWD_DKDV = 1, 2
CP_BWD_MAX_CHUNKS = 2

STATUS_NAMES = {0: "CP_OK", 1: "CP_ERR_INVALID_ARG", 2: "CP_ERR_UNSUPPORTED", 3: "CP_ERR_ALIGNMENT",
                4: "CP_ERR_WORKSPACE", 5: "CP_ERR_CUDA"}

EXPORTS = [
    "cp_last_error_string", "cp_version", "cp_block_attn_fwd", "cp_lse_merge",
    "cp_ring_attn_workspace_size", "cp_ring_attn_fwd", "cp_ulysses_permute", "cp_zigzag_reorder",
    "cp_ulysses_attn_workspace_size", "cp_ulysses_attn_fwd", "cp_ring_schedule", "cp_count_live_pairs",
    "cp_device_error", "cp_kernel_launch_count", "cp_set_profile_events",
    "cp_ring_attn_fwd_noalloc", "cp_selftest_wait_timeout", "cp_striped_reorder",
    "cp_usp_attn_workspace_size", "cp_usp_attn_fwd", "cp_ring_attn_bwd_workspace_size", "cp_ring_attn_bwd",
    "cp_usp_attn_bwd_workspace_size", "cp_usp_attn_bwd", "cp_ulysses_attn_bwd_workspace_size", "cp_ulysses_attn_bwd",
    "cp_head_block_split", "cp_attn_bwd_prep", "cp_block_attn_bwd",
]


class cp_chunk(ctypes.Structure):
    _fields_ = [("start", ctypes.c_int32), ("len", ctypes.c_int32)]


class CpError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m context_exact_attention_step_b200.build` "
            "(or __graft_entry__.build()); there is no non-CUDA fallback")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    P32 = ctypes.POINTER(ctypes.c_int32)
    P64 = ctypes.POINTER(ctypes.c_int64)
    L.cp_last_error_string.restype = ctypes.c_char_p
    L.cp_last_error_string.argtypes = []
    L.cp_version.restype = ctypes.c_char_p
    L.cp_version.argtypes = []
    L.cp_block_attn_fwd.restype = i32
    L.cp_block_attn_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.POINTER(cp_chunk), i32,
                                    ctypes.POINTER(cp_chunk), i32, i32, vp, i32, f32, vp, vp, vp]
    L.cp_lse_merge.restype = i32
    L.cp_lse_merge.argtypes = [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32, i32, vp, vp, vp, vp]
    L.cp_ring_attn_workspace_size.restype = i32
    L.cp_ring_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P32, i32,
                                              ctypes.POINTER(ctypes.c_size_t)]
    L.cp_ring_attn_fwd.restype = i32
    L.cp_ring_attn_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, P32, vp, i32, f32, vp, vp,
                                   vp, ctypes.c_size_t, vp]
    L.cp_ring_attn_fwd_noalloc.restype = i32
    L.cp_ring_attn_fwd_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, P32, vp, i32, f32,
                                           vp, vp, vp]
    L.cp_ulysses_permute.restype = i32
    L.cp_ulysses_permute.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.cp_striped_reorder.restype = i32
    L.cp_striped_reorder.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp]
    L.cp_head_block_split.restype = i32
    L.cp_head_block_split.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp]
    L.cp_attn_bwd_prep.restype = i32
    L.cp_attn_bwd_prep.argtypes = [vp, vp, vp, i32, i32, i32, vp, vp, vp]
    L.cp_block_attn_bwd.restype = i32
    L.cp_block_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.POINTER(cp_chunk), i32,
                                    ctypes.POINTER(cp_chunk), i32, i32, vp, i32, f32, vp, vp, vp, i32, i32, vp]
    L.cp_zigzag_reorder.restype = i32
    L.cp_zigzag_reorder.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp]
    L.cp_ulysses_attn_workspace_size.restype = i32
    L.cp_ulysses_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    L.cp_ulysses_attn_fwd.restype = i32
    L.cp_ulysses_attn_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, ctypes.c_size_t,
                                      vp]
    L.cp_usp_attn_workspace_size.restype = i32
    L.cp_usp_attn_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P32, i32,
                                             ctypes.POINTER(ctypes.c_size_t)]
    L.cp_usp_attn_fwd.restype = i32
    L.cp_usp_attn_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, P32, vp, i32, f32, vp, vp,
                                  vp, ctypes.c_size_t, vp]
    L.cp_ring_attn_bwd_workspace_size.restype = i32
    L.cp_ring_attn_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, P32, i32,
                                                  ctypes.POINTER(ctypes.c_size_t)]
    L.cp_ring_attn_bwd.restype = i32
    L.cp_ring_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, P32, vp, i32, f32,
                                   vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.cp_usp_attn_bwd_workspace_size.restype = i32
    L.cp_usp_attn_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, P32, i32,
                                                 ctypes.POINTER(ctypes.c_size_t)]
    L.cp_usp_attn_bwd.restype = i32
    L.cp_usp_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, P32, vp, i32, f32,
                                  vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.cp_ulysses_attn_bwd_workspace_size.restype = i32
    L.cp_ulysses_attn_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    L.cp_ulysses_attn_bwd.restype = i32
    L.cp_ulysses_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, vp, vp, vp, vp,
                                      ctypes.c_size_t, vp]
    L.cp_ring_schedule.restype = i32
    L.cp_ring_schedule.argtypes = [i32, i32, i32, i32, P32, i32, P32, P32, P32, P64]
    L.cp_count_live_pairs.restype = i32
    L.cp_count_live_pairs.argtypes = [i32, i32, P32, i32, P64]
    L.cp_kernel_launch_count.restype = i32
    L.cp_kernel_launch_count.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
    L.cp_set_profile_events.restype = i32
    L.cp_set_profile_events.argtypes = [vp, vp, vp]
    L.cp_selftest_wait_timeout.restype = i32
    L.cp_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    L.cp_device_error.restype = i32
    L.cp_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    _lib = L
    return L


def check(status):
    if status != CP_OK:
        raise CpError(status, lib().cp_last_error_string().decode(errors="replace"))
