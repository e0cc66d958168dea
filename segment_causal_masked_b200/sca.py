"""Python binding of libsca (include/sca.h): argument marshalling only.

Every function forwards to the C ABI of the same name (without the ``sca_``
prefix). Device buffers are passed as raw addresses: anything with a
``data_ptr()`` method (a torch tensor) or a plain ``int``. Streams are
``cudaStream_t`` handles as ints, or a ``torch.cuda.Stream``; ``None`` means
torch's current stream on the current device.

The module refuses to import when ``libsca.so`` is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Iterable, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsca.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m segment_causal_masked_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

HEAD_DIM = 128
TILE = 128
MAX_ACTIONS = 32
TEXTQ_OWN_TAIL, TEXTQ_FULL_SEGMENT = 0, 1
TILE_EMPTY, TILE_PARTIAL, TILE_FULL = 0, 1, 2
CAM_ALL, CAM_OWN_FRAME, CAM_UP_TO_FRAME = 0, 1, 2
MAX_CAMERA_TOKENS = 64
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED = 0, -1, -2, -3
ERR_CAPACITY, ERR_CUDA, ERR_DEVICE_TIMEOUT, ERR_MISMATCH = -4, -5, -6, -7

EXPORTED = (
    "sca_metadata_create", "sca_build_segment_mask_metadata",
    "sca_build_segment_mask_metadata_ex", "sca_metadata_get_counts",
    "sca_metadata_get_schedule", "sca_metadata_get_descriptors", "sca_metadata_upload",
    "sca_metadata_get_bwd_schedule",
    "sca_metadata_destroy", "sca_kv_cache_create", "sca_kv_cache_create_int8",
    "sca_kv_cache_append",
    "sca_kv_cache_truncate", "sca_kv_cache_get", "sca_kv_cache_destroy",
    "sca_action_causal_attn_fwd", "sca_action_causal_attn_fwd_static_ws",
    "sca_attn_workspace_bytes", "sca_attn_plan", "sca_attn_plan_for_sms",
    "sca_attn_int8_scratch_bytes",
    "sca_action_causal_attn_bwd", "sca_attn_bwd_workspace_bytes", "sca_camera_cross_attn",
    "sca_set_split_override", "sca_set_pipeline_timeout_ns",
    "sca_last_error", "sca_read_device_status", "sca_debug_bounded_wait",
)


class ScaError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"libsca error {code}: {message}")
        self.code = code


class sca_mask_options(ctypes.Structure):
    _fields_ = [("textq_policy", ctypes.c_int32), ("history_segments", ctypes.c_int32),
                ("keep_blocks", ctypes.c_void_p), ("keep_blocks_len", ctypes.c_int64)]


class sca_segment(ctypes.Structure):
    _fields_ = [("num_frames", ctypes.c_int32), ("tokens_per_frame", ctypes.c_int32),
                ("head_len", ctypes.c_int32), ("num_actions", ctypes.c_int32),
                ("action_len", ctypes.POINTER(ctypes.c_int32)),
                ("action_begin", ctypes.POINTER(ctypes.c_int32)),
                ("action_end", ctypes.POINTER(ctypes.c_int32))]


_P = ctypes.c_void_p
_i32, _i64 = ctypes.c_int32, ctypes.c_int64
_pi32, _pi64 = ctypes.POINTER(_i32), ctypes.POINTER(_i64)
_SIGS = {
    "sca_metadata_create": [ctypes.POINTER(_P)],
    "sca_build_segment_mask_metadata": [_P, ctypes.POINTER(sca_segment), _i32,
                                        ctypes.POINTER(sca_segment), _i32, _i32],
    "sca_build_segment_mask_metadata_ex": [_P, ctypes.POINTER(sca_segment), _i32,
                                           ctypes.POINTER(sca_segment), _i32,
                                           ctypes.POINTER(sca_mask_options)],
    "sca_metadata_get_counts": [_P, _pi64, _pi64, _pi64, _pi32, _pi32, _pi64, _pi64, _pi64],
    "sca_metadata_get_schedule": [_P, ctypes.POINTER(_pi32), ctypes.POINTER(_pi32),
                                  ctypes.POINTER(ctypes.POINTER(ctypes.c_uint8))],
    "sca_metadata_get_bwd_schedule": [_P, ctypes.POINTER(_pi32),
                                      ctypes.POINTER(ctypes.POINTER(ctypes.c_uint32)),
                                      ctypes.POINTER(_pi32)],
    "sca_metadata_get_descriptors": [_P, ctypes.POINTER(ctypes.POINTER(ctypes.c_uint32)),
                                     ctypes.POINTER(ctypes.POINTER(ctypes.c_uint32))],
    "sca_metadata_upload": [_P, _P],
    "sca_metadata_destroy": [_P],
    "sca_kv_cache_create": [ctypes.POINTER(_P), _i32, _i32, _i64, _P, _P, _P],
    "sca_kv_cache_create_int8": [ctypes.POINTER(_P), _i32, _i32, _i64, _P, _P, _P, _P, _P],
    "sca_kv_cache_append": [_P, ctypes.POINTER(sca_segment), _P, _P, _P],
    "sca_kv_cache_truncate": [_P, _i32],
    "sca_kv_cache_get": [_P, _pi64, _pi32],
    "sca_kv_cache_destroy": [_P],
    "sca_action_causal_attn_fwd": [_P, _P, _i32, _P, _P, _P, _P, _P, ctypes.c_float, _P,
                                   ctypes.c_uint64, _P, _P],
    "sca_action_causal_attn_fwd_static_ws": [_P, _P, _i32, _P, _P, _P, _P, _P, ctypes.c_float,
                                             _P, _P],
    "sca_attn_workspace_bytes": [_P, _i32, ctypes.POINTER(ctypes.c_uint64)],
    "sca_attn_int8_scratch_bytes": [_P, _i32, ctypes.POINTER(ctypes.c_uint64)],
    "sca_action_causal_attn_bwd": [_P, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_float,
                                   _P, ctypes.c_uint64, _P, _P],
    "sca_attn_bwd_workspace_bytes": [_P, _i32, ctypes.POINTER(ctypes.c_uint64)],
    "sca_camera_cross_attn": [_P, _P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, ctypes.c_float, _P,
                              _P],
    "sca_attn_plan": [_P, _i32, _pi32, _pi32, _pi32],
    "sca_attn_plan_for_sms": [_P, _i32, _i32, _pi32, _pi32, _pi32, ctypes.POINTER(ctypes.c_uint64)],
    "sca_set_split_override": [_i32],
    "sca_set_pipeline_timeout_ns": [_i64],
    "sca_last_error": [],
    "sca_read_device_status": [_P, _P],
    "sca_debug_bounded_wait": [_P, _i64, _P],
}
for _name, _args in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = None if _name.endswith("_destroy") else (
        ctypes.c_char_p if _name == "sca_last_error" else ctypes.c_int)


def last_error() -> str:
    return (_lib.sca_last_error() or b"").decode()


def _check(rc: int) -> None:
    if rc != 0:
        raise ScaError(rc, last_error())


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


class _SegArray:
    """ctypes array of sca_segment built from objects with the layout fields
    (num_frames, tokens_per_frame, head_len, actions=[(length, begin, end)])."""

    def __init__(self, segments: Iterable):
        segs = list(segments)
        self.arr = (sca_segment * max(1, len(segs)))()
        self._keep = []
        for i, s in enumerate(segs):
            acts = [(int(a.length), int(a.begin), int(a.end)) if hasattr(a, "length") else
                    tuple(int(x) for x in a) for a in s.actions]
            n = len(acts)
            ln = (ctypes.c_int32 * max(1, n))(*[a[0] for a in acts])
            bg = (ctypes.c_int32 * max(1, n))(*[a[1] for a in acts])
            en = (ctypes.c_int32 * max(1, n))(*[a[2] for a in acts])
            self._keep += [ln, bg, en]
            self.arr[i] = sca_segment(int(s.num_frames), int(s.tokens_per_frame), int(s.head_len),
                                      n, ln, bg, en)
        self.n = len(segs)


# ---------------------------------------------------------------------------
# metadata
# ---------------------------------------------------------------------------

class Metadata:
    """Owns one ``sca_metadata`` handle."""

    def __init__(self):
        h = _P()
        _check(_lib.sca_metadata_create(ctypes.byref(h)))
        self.handle = h

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.sca_metadata_destroy(self.handle)
            self.handle = None

    def build(self, cached: Sequence, current: Sequence, textq_policy: int = TEXTQ_OWN_TAIL,
              history_segments: int = -1, keep_blocks=None):
        """``keep_blocks``: None, or a [query tiles, key tiles] array of bools
        / 0-1 bytes (a 0 drops that video-only key tile for that query tile)."""
        c, u = _SegArray(cached), _SegArray(current)
        if history_segments == -1 and keep_blocks is None:
            _check(_lib.sca_build_segment_mask_metadata(self.handle, c.arr, c.n, u.arr, u.n,
                                                        int(textq_policy)))
            return self
        keep = None
        if keep_blocks is not None:
            import numpy as np
            keep = np.ascontiguousarray(np.asarray(keep_blocks).astype(np.uint8).ravel())
        opt = sca_mask_options(int(textq_policy), int(history_segments),
                               keep.ctypes.data if keep is not None else None,
                               int(keep.size) if keep is not None else 0)
        _check(_lib.sca_build_segment_mask_metadata_ex(self.handle, c.arr, c.n, u.arr, u.n,
                                                       ctypes.byref(opt)))
        return self

    def counts(self) -> dict:
        a, nq, nc, nnz, nf, npart = (_i64() for _ in range(6))
        nqt, nkt = _i32(), _i32()
        _check(_lib.sca_metadata_get_counts(self.handle, ctypes.byref(a), ctypes.byref(nq),
                                            ctypes.byref(nc), ctypes.byref(nqt), ctypes.byref(nkt),
                                            ctypes.byref(nnz), ctypes.byref(nf), ctypes.byref(npart)))
        return {"unmasked_pairs": a.value, "n_queries": nq.value, "n_cache_keys": nc.value,
                "n_q_tiles": nqt.value, "n_kv_tiles": nkt.value, "nnz": nnz.value,
                "n_full": nf.value, "n_partial": npart.value}

    def schedule(self):
        """(row_ptr, kv_tile, flag) as numpy copies."""
        import numpy as np
        c = self.counts()
        rp, kt = _pi32(), _pi32()
        fl = ctypes.POINTER(ctypes.c_uint8)()
        _check(_lib.sca_metadata_get_schedule(self.handle, ctypes.byref(rp), ctypes.byref(kt),
                                              ctypes.byref(fl)))
        n = c["nnz"]
        row_ptr = np.ctypeslib.as_array(rp, shape=(c["n_q_tiles"] + 1,)).copy()
        kv = np.ctypeslib.as_array(kt, shape=(max(n, 1),))[:n].copy()
        flag = np.ctypeslib.as_array(fl, shape=(max(n, 1),))[:n].copy()
        return row_ptr, kv, flag

    def bwd_schedule(self):
        """(kt_ptr, kt_list, kt_order) of the backward's key-major schedule as
        numpy copies (empty arrays for a layout with a cache)."""
        import numpy as np
        c = self.counts()
        kp, ko = _pi32(), _pi32()
        kl = ctypes.POINTER(ctypes.c_uint32)()
        _check(_lib.sca_metadata_get_bwd_schedule(self.handle, ctypes.byref(kp), ctypes.byref(kl),
                                                  ctypes.byref(ko)))
        if not kp:
            return np.zeros(0, np.int32), np.zeros(0, np.uint32), np.zeros(0, np.int32)
        n_kt = c["n_kv_tiles"]
        kt_ptr = np.ctypeslib.as_array(kp, shape=(n_kt + 1,)).copy()
        nnz = int(kt_ptr[-1])
        kt_list = np.ctypeslib.as_array(kl, shape=(max(nnz, 1),))[:nnz].copy()
        kt_order = np.ctypeslib.as_array(ko, shape=(n_kt,)).copy()
        return kt_ptr, kt_list, kt_order

    def descriptors(self):
        """(key descriptors of the current keys [n], query descriptors [n, 2])."""
        import numpy as np
        n = self.counts()["n_queries"]
        kd = ctypes.POINTER(ctypes.c_uint32)()
        qd = ctypes.POINTER(ctypes.c_uint32)()
        _check(_lib.sca_metadata_get_descriptors(self.handle, ctypes.byref(kd), ctypes.byref(qd)))
        return (np.ctypeslib.as_array(kd, shape=(n,)).copy(),
                np.ctypeslib.as_array(qd, shape=(n, 2)).copy())

    def upload(self, stream=None):
        _check(_lib.sca_metadata_upload(self.handle, _stream(stream)))
        return self


def build_segment_mask_metadata(cached: Sequence, current: Sequence,
                                textq_policy: int = TEXTQ_OWN_TAIL,
                                md: Optional[Metadata] = None, history_segments: int = -1,
                                keep_blocks=None) -> Metadata:
    return (md or Metadata()).build(cached, current, textq_policy, history_segments,
                                    keep_blocks)


def build_for(problem, md: Optional[Metadata] = None) -> Metadata:
    """Metadata of a workloads.Problem (its policy, window and kept blocks)."""
    return build_segment_mask_metadata(problem.cached, problem.current, problem.textq_policy, md,
                                       getattr(problem, "history_segments", -1),
                                       getattr(problem, "keep_blocks", None))


def metadata_upload(md: Metadata, stream=None) -> Metadata:
    return md.upload(stream)


# ---------------------------------------------------------------------------
# KV cache
# ---------------------------------------------------------------------------

class KVCache:
    """Owns one ``sca_kv_cache`` handle over caller-owned device buffers:
    k_buf, v_buf bf16 [heads, capacity, 128]; desc_buf uint32/int32
    [round_up(capacity, 128)]. With ``k_scale`` and ``v_scale`` (fp32
    [heads, capacity]) the cache is INT8: k_buf, v_buf then hold int8 codes
    [heads, capacity, 128] (sca_kv_cache_create_int8). The buffers must
    outlive the cache."""

    def __init__(self, heads: int, capacity: int, k_buf, v_buf, desc_buf, k_scale=None,
                 v_scale=None):
        h = _P()
        self.int8 = k_scale is not None or v_scale is not None
        if self.int8:
            _check(_lib.sca_kv_cache_create_int8(ctypes.byref(h), int(heads), HEAD_DIM,
                                                 int(capacity), _ptr(k_buf), _ptr(v_buf),
                                                 _ptr(k_scale), _ptr(v_scale), _ptr(desc_buf)))
        else:
            _check(_lib.sca_kv_cache_create(ctypes.byref(h), int(heads), HEAD_DIM, int(capacity),
                                            _ptr(k_buf), _ptr(v_buf), _ptr(desc_buf)))
        self.handle = h
        self.heads = heads
        self.capacity = capacity
        self._bufs = (k_buf, v_buf, desc_buf, k_scale, v_scale)

    def __del__(self):
        if getattr(self, "handle", None):
            _lib.sca_kv_cache_destroy(self.handle)
            self.handle = None

    def append(self, segment, k, v, stream=None):
        s = _SegArray([segment])
        _check(_lib.sca_kv_cache_append(self.handle, s.arr, _ptr(k), _ptr(v), _stream(stream)))

    def truncate(self, n_segments: int):
        _check(_lib.sca_kv_cache_truncate(self.handle, int(n_segments)))

    def get(self):
        n, s = _i64(), _i32()
        _check(_lib.sca_kv_cache_get(self.handle, ctypes.byref(n), ctypes.byref(s)))
        return n.value, s.value

    @property
    def length(self) -> int:
        return self.get()[0]


def kv_cache_create(heads, capacity, k_buf, v_buf, desc_buf) -> KVCache:
    return KVCache(heads, capacity, k_buf, v_buf, desc_buf)


def kv_cache_create_int8(heads, capacity, k_codes, v_codes, k_scale, v_scale, desc_buf) -> KVCache:
    return KVCache(heads, capacity, k_codes, v_codes, desc_buf, k_scale, v_scale)


def kv_cache_append(cache: KVCache, segment, k, v, stream=None) -> None:
    cache.append(segment, k, v, stream)


def kv_cache_truncate(cache: KVCache, n_segments: int) -> None:
    cache.truncate(n_segments)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def action_causal_attn_fwd(cache: Optional[KVCache], md: Metadata, heads: int, q, k_cur, v_cur, o,
                           lse=None, softmax_scale: float = 128 ** -0.5, workspace=None,
                           workspace_bytes: Optional[int] = None, dev_status=None,
                           stream=None) -> None:
    """``workspace``: optional device scratch (a uint8 tensor, or an int
    address with ``workspace_bytes``) of at least ``attn_workspace_bytes``."""
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = int(workspace.numel() * workspace.element_size())
    _check(_lib.sca_action_causal_attn_fwd(cache.handle if cache is not None else None, md.handle,
                                           int(heads), _ptr(q), _ptr(k_cur), _ptr(v_cur), _ptr(o),
                                           _ptr(lse), float(softmax_scale), _ptr(workspace),
                                           int(workspace_bytes or 0), _ptr(dev_status),
                                           _stream(stream)))


STATIC_WORKSPACE_BYTES = 32 << 20


def action_causal_attn_fwd_static_ws(cache: Optional[KVCache], md: Metadata, heads: int, q,
                                     k_cur, v_cur, o, lse=None,
                                     softmax_scale: float = 128 ** -0.5, dev_status=None,
                                     stream=None) -> None:
    """Same result as ``action_causal_attn_fwd`` with a workspace, for callers
    that must not allocate: the key-split scratch comes from a fixed array of
    ``STATIC_WORKSPACE_BYTES`` inside the library (shared by all calls, so
    calls must not overlap on the GPU). An automatic split plan that needs
    more runs unsplit; a forced split (``set_split_override``) that needs
    more raises ``ScaError`` with ``ERR_CAPACITY``. The first call on a
    device looks the array up and should precede any stream capture."""
    _check(_lib.sca_action_causal_attn_fwd_static_ws(
        cache.handle if cache is not None else None, md.handle, int(heads), _ptr(q), _ptr(k_cur),
        _ptr(v_cur), _ptr(o), _ptr(lse), float(softmax_scale), _ptr(dev_status), _stream(stream)))


def attn_bwd_workspace_bytes(md: Metadata, heads: int) -> int:
    """Scratch bytes the backward needs (D and LSE·log2(e) per row)."""
    b = ctypes.c_uint64()
    _check(_lib.sca_attn_bwd_workspace_bytes(md.handle, int(heads), ctypes.byref(b)))
    return int(b.value)


def action_causal_attn_bwd(md: Metadata, heads: int, q, k, v, o, lse, d_o, dq, dk, dv,
                           softmax_scale: float = 128 ** -0.5, workspace=None,
                           workspace_bytes: Optional[int] = None, dev_status=None,
                           stream=None) -> None:
    """Gradients dq, dk, dv (written) of the forward for upstream gradient
    d_o; ``workspace``: a uint8 device tensor (or an int address with
    ``workspace_bytes``) of at least ``attn_bwd_workspace_bytes``."""
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = int(workspace.numel() * workspace.element_size())
    _check(_lib.sca_action_causal_attn_bwd(md.handle, int(heads), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk),
                                           _ptr(dv), float(softmax_scale), _ptr(workspace),
                                           int(workspace_bytes or 0), _ptr(dev_status),
                                           _stream(stream)))


def camera_cross_attn(q, k_cam, v_cam, x, out, q_frame=None, mode: int = CAM_ALL,
                      softmax_scale: float = 128 ** -0.5, dev_status=None, stream=None) -> None:
    """out = x + the camera cross-attention of queries ``q`` over one
    segment's camera tokens (see include/sca.h). ``q``, ``x``, ``out``: bf16
    [n_q, heads, 128] (``out`` may be ``x``); ``k_cam``, ``v_cam``: bf16
    [n_cam, heads, 128]; ``q_frame``: int32 [n_q] or None (SCA_CAM_ALL);
    ``dev_status``: device int32 or None."""
    n_q, heads = int(q.shape[0]), int(q.shape[1])
    if tuple(x.shape) != tuple(q.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("q, x and out must have the same shape [n_q, heads, 128]")
    if tuple(v_cam.shape) != tuple(k_cam.shape) or tuple(k_cam.shape[1:]) != (heads, HEAD_DIM):
        raise ValueError("k_cam and v_cam must be [n_cam, heads, 128]")
    _check(_lib.sca_camera_cross_attn(_ptr(q), _ptr(q_frame), _ptr(k_cam), _ptr(v_cam), _ptr(x),
                                      _ptr(out), n_q, int(k_cam.shape[0]), heads, int(mode),
                                      float(softmax_scale), _ptr(dev_status), _stream(stream)))


def attn_int8_scratch_bytes(md: Metadata, heads: int) -> int:
    """Extra workspace that lets an INT8-cache attention dequantise once into
    a bf16 copy (see include/sca.h)."""
    b = ctypes.c_uint64()
    _check(_lib.sca_attn_int8_scratch_bytes(md.handle, int(heads), ctypes.byref(b)))
    return int(b.value)


def attn_workspace_bytes(md: Metadata, heads: int) -> int:
    """Scratch bytes the attention's split plan needs on the current device."""
    b = ctypes.c_uint64()
    _check(_lib.sca_attn_workspace_bytes(md.handle, int(heads), ctypes.byref(b)))
    return int(b.value)


def attn_plan(md: Metadata, heads: int) -> dict:
    """The work split the next call would run (with enough workspace)."""
    a, b, c = _i32(), _i32(), _i32()
    _check(_lib.sca_attn_plan(md.handle, int(heads), ctypes.byref(a), ctypes.byref(b),
                              ctypes.byref(c)))
    return {"n_full": a.value, "n_split": b.value, "chunks": c.value}


def attn_plan_for_sms(md: Metadata, heads: int, sms: int) -> dict:
    """The work split for a device with ``sms`` SMs (no device needed), with
    the workspace bytes it takes."""
    a, b, c = _i32(), _i32(), _i32()
    w = ctypes.c_uint64()
    _check(_lib.sca_attn_plan_for_sms(md.handle, int(heads), int(sms), ctypes.byref(a),
                                      ctypes.byref(b), ctypes.byref(c), ctypes.byref(w)))
    return {"n_full": a.value, "n_split": b.value, "chunks": c.value, "workspace_bytes": w.value}


def set_split_override(chunks: int) -> None:
    """0 = automatic split plan, 1 = never split, k >= 2 = split the tail into
    k chunks; for calls made from the calling thread."""
    _check(_lib.sca_set_split_override(int(chunks)))


def read_device_status(dev_status, stream=None) -> int:
    """The status word after the stream's queued work: 0, else raises
    ``ScaError`` with the code a kernel stored there."""
    _check(_lib.sca_read_device_status(_ptr(dev_status), _stream(stream)))
    return OK


def set_pipeline_timeout_ns(ns: int) -> None:
    """Limit of the kernels' pipeline waits for calls from the calling thread
    (default 2 s; 0 exercises the abort path)."""
    _check(_lib.sca_set_pipeline_timeout_ns(int(ns)))


def debug_bounded_wait(dev_status, timeout_ns: int, stream=None) -> None:
    _check(_lib.sca_debug_bounded_wait(_ptr(dev_status), int(timeout_ns), _stream(stream)))
