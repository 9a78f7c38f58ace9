"""ctypes binding of libai_index.so: argument marshalling only.

Every function here forwards to the C entry point of the same name in
include/ai_index.h; all computation happens in the library's CUDA kernels.
Tensors are torch tensors on the device the handle was created on; torch
supplies device memory and the stream, nothing else.  There is no CPU
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libai_index.so")

AI_OK = 0
ERRORS = {
    -1: "AI_ERR_ARG", -2: "AI_ERR_OOM", -3: "AI_ERR_CAUSALITY", -4: "AI_ERR_DEVICE_CHECK",
    -5: "AI_ERR_TIMEOUT", -6: "AI_ERR_CUDA", -7: "AI_ERR_STATE",
}
AI_FP32, AI_BF16, AI_FP8E4M3 = 0, 1, 2
DTYPES = {"fp32": AI_FP32, "bf16": AI_BF16, "fp8": AI_FP8E4M3}

EXPORTED = [
    "ai_index_create", "ai_index_destroy", "ai_append_keys", "ai_seal", "ai_refit",
    "ai_publish", "ai_route_refine", "ai_select_exhaustive", "ai_sync", "ai_last_error",
    "ai_get_stats", "ai_export_index", "ai_debug_candidates", "ai_debug_scores",
    "ai_checkpoint", "ai_rollback", "ai_quantize_fp8", "ai_profile_enable", "ai_profile_read",
    "ai_kernel_launches", "ai_select_exhaustive_noalloc", "ai_debug_wait_timeout",
    "ai_route_refine_shard", "ai_merge_topk",
    "ai_debug_refine_kernel", "ai_refine_kernel_choice", "ai_debug_refine_split",
]
PHASES = ["route", "refine", "seal", "refit", "publish", "exh_scores", "exh_topk", "order"]


class AiConfig(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int32), ("H", ctypes.c_int32), ("key_dtype", ctypes.c_int32),
        ("q_dtype", ctypes.c_int32), ("n_sinks", ctypes.c_int32), ("window", ctypes.c_int32),
        ("clusters_per_window", ctypes.c_int32), ("cluster_cap", ctypes.c_int32),
        ("refit_period", ctypes.c_int32), ("refit_new_seeds", ctypes.c_int32),
        ("refit_seed_window", ctypes.c_int32), ("seal_iters", ctypes.c_int32),
        ("async_refit", ctypes.c_int32), ("max_query_chunk", ctypes.c_int32),
        ("max_budget", ctypes.c_int32), ("max_k", ctypes.c_int32),
        ("max_keys", ctypes.c_int64), ("seed", ctypes.c_uint64),
        ("encoder_weights_host", ctypes.POINTER(ctypes.c_float)),
        ("block_routing", ctypes.c_int32),
    ]


class AiStats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "n_keys", "n_sealed", "n_clusters", "n_versions", "n_refits", "refit_pending",
        "base_watermark", "last_refit_scanned", "last_refit_rechecked")]


class AiError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python ivf_top_key_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "ai_index_create": [ctypes.POINTER(AiConfig), vp, ctypes.POINTER(vp)],
        "ai_index_destroy": [vp],
        "ai_append_keys": [vp, vp, vp, i64],
        "ai_seal": [vp, ctypes.POINTER(i64)],
        "ai_refit": [vp, i32, i32, ctypes.POINTER(i64)],
        "ai_publish": [vp],
        "ai_route_refine": [vp, vp, vp, i64, i32, i32, i32, vp, vp],
        "ai_select_exhaustive": [vp, vp, vp, i64, i32, i32, vp, vp],
        "ai_sync": [vp],
        "ai_get_stats": [vp, ctypes.POINTER(AiStats)],
        "ai_export_index": [vp, vp, vp, vp, vp, vp, vp],
        "ai_debug_candidates": [vp, vp, vp, i64, i32, i32, vp, vp],
        "ai_debug_scores": [vp, vp, vp, i64, i32, vp],
        "ai_checkpoint": [vp],
        "ai_rollback": [vp],
        "ai_quantize_fp8": [vp, i64, i32, vp, vp, vp],
        "ai_profile_enable": [vp, ctypes.c_int],
        "ai_profile_read": [vp, vp, vp],
        "ai_select_exhaustive_noalloc": [vp, i32, i64, i32, i32, vp, vp, i64, i32, i32, vp, vp, vp, vp],
        "ai_route_refine_shard": [vp, vp, vp, i64, i32, i32, i32, i32, i32, vp, vp],
        "ai_merge_topk": [vp, vp, i32, i32, i32, vp, vp, vp],
        "ai_debug_wait_timeout": [i32, ctypes.POINTER(i32), vp],
        "ai_debug_refine_kernel": [vp, i32],
        "ai_debug_refine_split": [vp, i32],
        "ai_refine_kernel_choice": [vp, i32, ctypes.POINTER(i32)],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.ai_kernel_launches.argtypes = []
    lib.ai_kernel_launches.restype = ctypes.c_longlong
    lib.ai_last_error.argtypes = []
    lib.ai_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load()


def _check(rc: int):
    if rc != AI_OK:
        raise AiError(rc, _lib.ai_last_error().decode(errors="replace"))


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---- the C entry points, same names -------------------------------------

def ai_index_create(cfg: AiConfig, stream=None) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(_lib.ai_index_create(ctypes.byref(cfg), _stream(stream), ctypes.byref(h)))
    return h


def ai_index_destroy(h):
    _check(_lib.ai_index_destroy(h))


def ai_append_keys(h, keys, scales=None):
    _check(_lib.ai_append_keys(h, _ptr(keys), _ptr(scales), keys.shape[0]))


def ai_seal(h) -> int:
    v = ctypes.c_int64()
    _check(_lib.ai_seal(h, ctypes.byref(v)))
    return v.value


def ai_refit(h, n_new_seeds: int = 0, seed_window: int = 0) -> int:
    v = ctypes.c_int64()
    _check(_lib.ai_refit(h, n_new_seeds, seed_window, ctypes.byref(v)))
    return v.value


def ai_publish(h):
    _check(_lib.ai_publish(h))


def ai_route_refine(h, q, w, pos0: int, k: int, C: int, out, out_scores=None):
    _check(_lib.ai_route_refine(h, _ptr(q), _ptr(w), pos0, q.shape[0], k, C, _ptr(out), _ptr(out_scores)))
    return out


def ai_select_exhaustive(h, q, w, pos0: int, k: int, out, out_scores=None):
    _check(_lib.ai_select_exhaustive(h, _ptr(q), _ptr(w), pos0, q.shape[0], k, _ptr(out), _ptr(out_scores)))
    return out


def ai_sync(h):
    _check(_lib.ai_sync(h))


def ai_get_stats(h) -> dict:
    st = AiStats()
    _check(_lib.ai_get_stats(h, ctypes.byref(st)))
    return {n: getattr(st, n) for n, _ in AiStats._fields_}


def ai_export_index(h, d: int) -> dict:
    st = ai_get_stats(h)
    nC, nv = st["n_clusters"], st["n_versions"]
    import numpy as np
    offsets = np.zeros(nC + 1, dtype=np.int32)
    _check(_lib.ai_export_index(h, offsets.ctypes.data_as(ctypes.c_void_p), None, None, None, None, None))
    members = np.zeros(max(int(offsets[-1]), 1), dtype=np.int32)
    reps = np.zeros((max(nC, 1), d), dtype=np.uint16)
    cents = np.zeros((max(nC, 1), d), dtype=np.float64)
    vnc = np.zeros(max(nv, 1), dtype=np.int64)
    vnv = np.zeros(max(nv, 1), dtype=np.int64)
    c = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(_lib.ai_export_index(h, c(offsets), c(members), c(reps), c(cents), c(vnc), c(vnv)))
    return {"offsets": offsets, "members": members[:int(offsets[-1])], "reps_bf16": reps[:nC],
            "centroids": cents[:nC], "version_nc": vnc[:nv], "version_nv": vnv[:nv]}


def ai_debug_candidates(h, q, w, pos0: int, C: int, cand, cluster_scores=None):
    _check(_lib.ai_debug_candidates(h, _ptr(q), _ptr(w), pos0, q.shape[0], C, _ptr(cand), _ptr(cluster_scores)))
    return cand


def ai_debug_scores(h, q, w, pos0: int, out):
    _check(_lib.ai_debug_scores(h, _ptr(q), _ptr(w), pos0, q.shape[0], _ptr(out)))
    return out


def ai_checkpoint(h):
    _check(_lib.ai_checkpoint(h))


def ai_rollback(h):
    _check(_lib.ai_rollback(h))


def ai_quantize_fp8(keys_bf16, codes, scales, stream=None):
    _check(_lib.ai_quantize_fp8(_ptr(keys_bf16), keys_bf16.shape[0], keys_bf16.shape[1],
                                _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def ai_profile_enable(h, enable: bool = True):
    _check(_lib.ai_profile_enable(h, int(enable)))


def ai_profile_read(h) -> dict:
    import numpy as np
    ms = np.zeros(len(PHASES), dtype=np.float64)
    n = np.zeros(len(PHASES), dtype=np.int64)
    _check(_lib.ai_profile_read(h, ms.ctypes.data_as(ctypes.c_void_p), n.ctypes.data_as(ctypes.c_void_p)))
    return {p: (float(ms[i]), int(n[i])) for i, p in enumerate(PHASES)}


def ai_kernel_launches() -> int:
    return int(_lib.ai_kernel_launches())


def ai_select_exhaustive_noalloc(keys, key_dtype: int, q, w, pos0: int, k: int, out,
                                 out_scores=None, status=None, stream=None):
    """Exhaustive selection without any device allocation (see the header).
    status: None or a 1-element int32 device tensor for the device flags."""
    n, d = keys.shape[0], keys.shape[1]
    _check(_lib.ai_select_exhaustive_noalloc(_ptr(keys), key_dtype, n, d, q.shape[1], _ptr(q), _ptr(w),
                                             pos0, q.shape[0], k, _ptr(out), _ptr(out_scores),
                                             _ptr(status), _stream(stream)))
    return out


def ai_route_refine_shard(h, q, w, pos0: int, k: int, C: int, shard: int, n_shards: int, out, out_scores):
    _check(_lib.ai_route_refine_shard(h, _ptr(q), _ptr(w), pos0, q.shape[0], k, C, shard, n_shards,
                                      _ptr(out), _ptr(out_scores)))
    return out, out_scores


def ai_merge_topk(ids, scores, k: int, out, out_scores=None, stream=None):
    """ids / scores: [n_parts, T, k] device tensors."""
    _check(_lib.ai_merge_topk(_ptr(ids), _ptr(scores), ids.shape[0], ids.shape[1], k, _ptr(out),
                              _ptr(out_scores), _stream(stream)))
    return out


def ai_debug_wait_timeout(spin_limit: int, stream=None) -> int:
    """Bounded wait on a barrier nothing completes; returns the device status
    flags it recorded (bit 0 = timeout)."""
    st = ctypes.c_int32(0)
    _check(_lib.ai_debug_wait_timeout(spin_limit, ctypes.byref(st), _stream(stream)))
    return st.value


def ai_debug_refine_kernel(h, kernel: int):
    """Select the tensor-core refine variant (0 auto, 1 sequential with the
    list in shared memory, 2 sequential with a global list, 3 pipelined,
    4 pipelined with one TMEM score buffer)."""
    _check(_lib.ai_debug_refine_kernel(h, kernel))


def ai_debug_refine_split(h, split: int):
    """Parts per query of small chunks on the pipelined refine (0 = by
    chunk size, 1 = never divide, 2..8 = at most that many)."""
    _check(_lib.ai_debug_refine_split(h, split))


def ai_refine_kernel_choice(h, C: int) -> int:
    """Refine kernel the library launches for budget C (0 = fp32 SIMT path,
    1 / 2 = one query per CTA, 3 / 4 = pipelined with two / one score
    buffers)."""
    v = ctypes.c_int32()
    _check(_lib.ai_refine_kernel_choice(h, C, ctypes.byref(v)))
    return v.value


def ai_last_error() -> str:
    return _lib.ai_last_error().decode(errors="replace")
