"""Exact blockwise (ring) attention on one B200 - Python binding of libra_b200.so.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/ra.h``.  PyTorch supplies device
memory and the current CUDA stream.  There is no CPU fallback: importing this
package fails loudly when the library is missing, and every call raises
``RAError`` on a non-OK status.

Names follow the C ABI (``ra_block_attn``, ``ra_merge_partial``,
``ra_ring_attention`` ...).  Layouts: q/out ``[B, S, Hq, D]``, k/v
``[B, S, Hkv, D]``, lse ``[B, S, Hq]``, all contiguous.

``ring`` (a submodule, imported on demand) runs the sequence-parallel form
across ranks, one block of the sequence per rank, on top of these calls and
torch.distributed point-to-point messages.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# RA_DEBUG_BOUNDS=1 selects the checked build (every run-time-indexed global
# access checked on the device; see ra_debug_build in include/ra.h).
DEBUG_BOUNDS = os.environ.get("RA_DEBUG_BOUNDS", "0") == "1"
LIB_PATH = os.path.join(_PKG, "libra_b200_debug.so" if DEBUG_BOUNDS else "libra_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python blockwise_exact_attention_block_b200/build.py"
        f"{' --debug-bounds' if DEBUG_BOUNDS else ''}`")

_lib = ctypes.CDLL(LIB_PATH)

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_WORKSPACE = 0, 1, 2, 3
RA_ERR_CUDA, RA_ERR_TIMEOUT, RA_ERR_DEVICE_BOUNDS = 4, 5, 6
RA_F32, RA_BF16 = 0, 1
RA_PART_CONTIGUOUS, RA_PART_ZIGZAG = 0, 1
RA_ORDER_RING, RA_ORDER_TOKENRING = 0, 1
RA_SCHED_AUTO, RA_SCHED_UNFUSED, RA_SCHED_EPILOGUE_FUSED, RA_SCHED_PERSISTENT = 0, 1, 2, 3

PARTITIONS = {"contiguous": RA_PART_CONTIGUOUS, "zigzag": RA_PART_ZIGZAG}
ORDERS = {"ring": RA_ORDER_RING, "tokenring": RA_ORDER_TOKENRING}
SCHEDS = {"auto": RA_SCHED_AUTO, "unfused": RA_SCHED_UNFUSED, "fused": RA_SCHED_EPILOGUE_FUSED,
          "persistent": RA_SCHED_PERSISTENT}

EXPORTED = ["ra_block_attn", "ra_block_attn_merge", "ra_merge_partial", "ra_merge_partials", "ra_ring_attention",
            "ra_ring_attention_workspace", "ra_zigzag_permute", "ra_get_device_status",
            "ra_status_string", "ra_version", "ra_ring_attention_noalloc", "ra_noalloc_scratch_bytes",
            "ra_decode_attention", "ra_decode_workspace", "ra_decode_splits", "ra_ring_attention_backward",
            "ra_ring_attention_backward_workspace", "ra_debug_build", "ra_get_bounds_record",
            "ra_set_cta_timeline"]

RA_TIMELINE_ATTN_FWD, RA_TIMELINE_BWD_DKV, RA_TIMELINE_BWD_DQ = 0, 1, 2
TIMELINE_KERNELS = {"attn_fwd": RA_TIMELINE_ATTN_FWD, "bwd_dkv": RA_TIMELINE_BWD_DKV, "bwd_dq": RA_TIMELINE_BWD_DQ}


class ra_options(ctypes.Structure):
    _fields_ = [("order", ctypes.c_int), ("sched", ctypes.c_int), ("attn_event_begin", ctypes.c_void_p),
                ("attn_event_end", ctypes.c_void_p), ("tiling", ctypes.c_int), ("fault_inject", ctypes.c_int)]


TILINGS = {"auto": 0, "row_pairs": 1, "kv_split": 2, "cluster2": 3}


_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_lib.ra_block_attn.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]
_lib.ra_block_attn.restype = _i
_lib.ra_block_attn_merge.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]
_lib.ra_block_attn_merge.restype = _i
_lib.ra_merge_partial.argtypes = [_vp, _vp, _vp, _vp, _i64, _i, _vp]
_lib.ra_merge_partial.restype = _i
_lib.ra_merge_partials.argtypes = [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp, _vp, _i64, _i, _vp]
_lib.ra_merge_partials.restype = _i
_lib.ra_ring_attention.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _sz,
                                   ctypes.POINTER(ra_options), _vp]
_lib.ra_ring_attention.restype = _i
_lib.ra_ring_attention_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(ra_options)]
_lib.ra_ring_attention_workspace.restype = _sz
_lib.ra_ring_attention_noalloc.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _i, _vp,
                                           ctypes.POINTER(ra_options), _vp]
_lib.ra_ring_attention_noalloc.restype = _i
_lib.ra_noalloc_scratch_bytes.argtypes = []
_lib.ra_noalloc_scratch_bytes.restype = _sz
_lib.ra_zigzag_permute.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
_lib.ra_zigzag_permute.restype = _i
_lib.ra_get_device_status.argtypes = [_vp]
_lib.ra_get_device_status.restype = _i
_lib.ra_status_string.argtypes = [_i]
_lib.ra_status_string.restype = ctypes.c_char_p
_lib.ra_version.argtypes = []
_lib.ra_version.restype = ctypes.c_char_p
_lib.ra_decode_attention.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _sz, _vp]
_lib.ra_decode_attention.restype = _i
_lib.ra_decode_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i]
_lib.ra_decode_workspace.restype = _sz
_lib.ra_decode_splits.argtypes = [_i, _i, _i, _i, _i, _i, _i]
_lib.ra_decode_splits.restype = _i
_lib.ra_ring_attention_backward.argtypes = [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                                            _vp, _vp, _vp, _vp, _sz, ctypes.POINTER(ra_options), _vp]
_lib.ra_ring_attention_backward.restype = _i
_lib.ra_ring_attention_backward_workspace.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i]
_lib.ra_ring_attention_backward_workspace.restype = _sz
_lib.ra_debug_build.argtypes = []
_lib.ra_debug_build.restype = _i
_lib.ra_get_bounds_record.argtypes = [ctypes.POINTER(ctypes.c_int64)]
_lib.ra_get_bounds_record.restype = _i
_lib.ra_set_cta_timeline.argtypes = [_vp, _i64, _i]
_lib.ra_set_cta_timeline.restype = _i


class RAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {ra_status_string(status)} ({status})")


def _check(status: int, what: str) -> None:
    if status != RA_OK:
        raise RAError(status, what)


def ra_status_string(status: int) -> str:
    return _lib.ra_status_string(status).decode()


def ra_version() -> str:
    return _lib.ra_version().decode()


def ra_debug_build() -> bool:
    """True when the loaded library is the checked build (RA_DEBUG_BOUNDS)."""
    return _lib.ra_debug_build() == 1


def ra_get_bounds_record() -> tuple[int, int, int]:
    """(source line, index, limit) of the first failed device index check
    since the last read (zeros if none), then cleared."""
    rec = (ctypes.c_int64 * 3)()
    _check(_lib.ra_get_bounds_record(rec), "ra_get_bounds_record")
    return int(rec[0]), int(rec[1]), int(rec[2])


def ra_set_cta_timeline(records: torch.Tensor | None, kernel: str = "attn_fwd") -> None:
    """Per-CTA timeline of one kernel's following launches (tracing).

    records: a contiguous int64 CUDA tensor [max_ctas, 4] that receives, per
    CTA, (start ns, end ns, SM id, work units); None turns the timeline off.
    kernel: "attn_fwd", "bwd_dkv" or "bwd_dq".  The tensor must stay alive
    until the launches that write it have completed."""
    if kernel not in TIMELINE_KERNELS:
        raise ValueError(f"unknown kernel {kernel!r}")
    if records is None:
        _check(_lib.ra_set_cta_timeline(None, 0, TIMELINE_KERNELS[kernel]), "ra_set_cta_timeline")
        return
    if records.dtype != torch.int64 or records.dim() != 2 or records.shape[1] != 4:
        raise ValueError("records must be an int64 tensor [max_ctas, 4]")
    _check(_lib.ra_set_cta_timeline(_ptr(records), records.shape[0], TIMELINE_KERNELS[kernel]),
           "ra_set_cta_timeline")


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return RA_BF16
    if dt == torch.float32:
        return RA_F32
    raise ValueError(f"unsupported dtype {dt}")


def _opts(order: str, sched: str, events=None, tiling: str = "auto", fault_inject: int = 0) -> ra_options:
    o = ra_options(ORDERS[order], SCHEDS[sched], None, None, TILINGS[tiling], fault_inject)
    if events is not None:
        for ev in events:
            if ev.cuda_event == 0:  # torch creates the CUDA event on its first record
                ev.record()
        o.attn_event_begin = events[0].cuda_event
        o.attn_event_end = events[1].cuda_event
    return o


def ra_block_attn(q, k, v, S: int, n_blocks: int, q_block: int, kv_block: int, causal: bool,
                  partition: str = "contiguous", block_out=None, block_lse=None, stream=None):
    """One query block [B, L, Hq, D] against one KV block [B, L, Hkv, D] (bf16).

    Returns (block_out fp32 [B, L, Hq, D], block_lse fp32 [B, L, Hq])."""
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    if block_out is None:
        block_out = torch.empty((B, L, Hq, D), dtype=torch.float32, device=q.device)
    if block_lse is None:
        block_lse = torch.empty((B, L, Hq), dtype=torch.float32, device=q.device)
    _check(_lib.ra_block_attn(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, S, n_blocks, q_block, kv_block,
                              Hq, Hkv, D, int(bool(causal)), PARTITIONS[partition], _ptr(block_out),
                              _ptr(block_lse), _stream(stream)), "ra_block_attn")
    return block_out, block_lse


def ra_block_attn_merge(q, k, v, S: int, n_blocks: int, q_block: int, kv_block: int, causal: bool, out, lse,
                        partition: str = "contiguous", stream=None):
    """One query block [B, L, Hq, D] against one KV block [B, L, Hkv, D] (bf16),
    folded by the merge rule into the running (out fp32 [B, L, Hq, D],
    lse fp32 [B, L, Hq]) in place.  Start from out = 0, lse = -inf."""
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    _check(_lib.ra_block_attn_merge(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, S, n_blocks, q_block,
                                    kv_block, Hq, Hkv, D, int(bool(causal)), PARTITIONS[partition], _ptr(out),
                                    _ptr(lse), _stream(stream)), "ra_block_attn_merge")
    return out, lse


def ra_merge_partial(out, lse, block_out, block_lse, stream=None):
    """In place: (out, lse) <- merge rule with (block_out, block_lse); fp32, rows x D."""
    D = out.shape[-1]
    rows = lse.numel()
    _check(_lib.ra_merge_partial(_ptr(out), _ptr(lse), _ptr(block_out), _ptr(block_lse), rows, D,
                                 _stream(stream)), "ra_merge_partial")
    return out, lse


def ra_merge_partials(outs, lses, out=None, lse=None, stream=None):
    """Fold k partials (lists of fp32 tensors) into one (out, lse) in a single pass."""
    k = len(outs)
    D = outs[0].shape[-1]
    rows = lses[0].numel()
    if out is None:
        out = torch.empty_like(outs[0])
    if lse is None:
        lse = torch.empty_like(lses[0])
    po = (_vp * k)(*[_ptr(t) for t in outs])
    pl = (_vp * k)(*[_ptr(t) for t in lses])
    _check(_lib.ra_merge_partials(po, pl, k, _ptr(out), _ptr(lse), rows, D, _stream(stream)), "ra_merge_partials")
    return out, lse


def ra_ring_attention_workspace(B, S, Hq, D, n_blocks, gqa_groups, partition="contiguous",
                                in_dtype=torch.bfloat16, order="ring", sched="auto",
                                out_dtype=torch.float32) -> int:
    o = _opts(order, sched)
    n = _lib.ra_ring_attention_workspace(B, S, Hq, D, n_blocks, gqa_groups, PARTITIONS[partition],
                                         _dtype_code(in_dtype), _dtype_code(out_dtype), ctypes.byref(o))
    if n == ctypes.c_size_t(-1).value:
        raise RAError(RA_ERR_INVALID_ARG, "ra_ring_attention_workspace")
    return n


def ra_ring_attention(q, k, v, n_blocks: int, causal: bool, partition: str = "contiguous",
                      gqa_groups: int | None = None, out=None, out_dtype=torch.float32, lse=None,
                      workspace=None, order: str = "ring", sched: str = "auto", stream=None,
                      attn_events=None, tiling: str = "auto", fault_inject: int = 0):
    """The whole method on one GPU.  Returns (out [B, S, Hq, D], lse fp32 [B, S, Hq]).

    attn_events: optional pair of torch.cuda.Event recorded around the
    block-attention launches inside the call.  fault_inject=1 is for testing
    the failure path only (see ra_options in include/ra.h)."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if gqa_groups is None:
        gqa_groups = Hq // Hkv
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device)
    need = ra_ring_attention_workspace(B, S, Hq, D, n_blocks, gqa_groups, partition, q.dtype, order, sched,
                                       out.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    o = _opts(order, sched, attn_events, tiling, fault_inject)
    _check(_lib.ra_ring_attention(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, S, Hq, D, n_blocks,
                                  int(bool(causal)), PARTITIONS[partition], gqa_groups, _ptr(out),
                                  _dtype_code(out.dtype), _ptr(lse), _ptr(workspace), ws_bytes, ctypes.byref(o),
                                  _stream(stream)), "ra_ring_attention")
    return out, lse


def ra_ring_attention_noalloc(q, k, v, n_blocks: int, causal: bool, partition: str = "contiguous",
                              gqa_groups: int | None = None, out=None, out_dtype=torch.float32, lse=None,
                              order: str = "ring", sched: str = "auto", stream=None, tiling: str = "auto"):
    """ra_ring_attention with its scratch in the library's fixed device array.

    For callers that may not allocate device memory at call time (their
    framework owns the GPU's memory pool, or cudaMalloc's implicit device
    synchronisation is not acceptable).  Pass `out` and `lse` to keep this
    wrapper from allocating them.  Calls that need more than
    ra_noalloc_scratch_bytes() of scratch raise RAError(RA_ERR_WORKSPACE);
    calls that overlap on the GPU share the one scratch array and race."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if gqa_groups is None:
        gqa_groups = Hq // Hkv
    if out is None:
        out = torch.empty((B, S, Hq, D), dtype=out_dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device)
    o = _opts(order, sched, None, tiling)
    _check(_lib.ra_ring_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, S, Hq, D, n_blocks,
                                          int(bool(causal)), PARTITIONS[partition], gqa_groups, _ptr(out),
                                          _dtype_code(out.dtype), _ptr(lse), ctypes.byref(o), _stream(stream)),
           "ra_ring_attention_noalloc")
    return out, lse


def ra_ring_attention_backward_workspace(B, S, Hq, D, n_blocks, gqa_groups, partition="contiguous",
                                         in_dtype=torch.bfloat16) -> int:
    n = _lib.ra_ring_attention_backward_workspace(B, S, Hq, D, n_blocks, gqa_groups, PARTITIONS[partition],
                                                  _dtype_code(in_dtype))
    if n == ctypes.c_size_t(-1).value:
        raise RAError(RA_ERR_INVALID_ARG, "ra_ring_attention_backward_workspace")
    return n


def ra_ring_attention_backward(q, k, v, out, lse, dout, n_blocks: int, causal: bool, partition: str = "contiguous",
                               gqa_groups: int | None = None, dq=None, dk=None, dv=None, workspace=None,
                               order: str = "ring", stream=None, attn_events=None):
    """Gradients of ra_ring_attention.  q, k, v, dout share one dtype (bf16 or
    fp32); out, lse are the forward's results.  Returns fp32 (dq, dk, dv).

    attn_events: optional pair of torch.cuda.Event recorded around the two
    tensor-core launches (dK/dV, then dQ) inside the call."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if gqa_groups is None:
        gqa_groups = Hq // Hkv
    if dout.dtype != q.dtype:
        raise ValueError("dout must have the dtype of q, k and v")
    if dq is None:
        dq = torch.empty((B, S, Hq, D), dtype=torch.float32, device=q.device)
    if dk is None:
        dk = torch.empty((B, S, Hkv, D), dtype=torch.float32, device=q.device)
    if dv is None:
        dv = torch.empty((B, S, Hkv, D), dtype=torch.float32, device=q.device)
    need = ra_ring_attention_backward_workspace(B, S, Hq, D, n_blocks, gqa_groups, partition, q.dtype)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    o = _opts(order, "auto", attn_events)
    _check(_lib.ra_ring_attention_backward(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), _ptr(out),
                                           _dtype_code(out.dtype), _ptr(lse), _ptr(dout), B, S, Hq, D, n_blocks,
                                           int(bool(causal)), PARTITIONS[partition], gqa_groups, _ptr(dq), _ptr(dk),
                                           _ptr(dv), _ptr(workspace), ws_bytes, ctypes.byref(o), _stream(stream)),
           "ra_ring_attention_backward")
    return dq, dk, dv


def ra_noalloc_scratch_bytes() -> int:
    return _lib.ra_noalloc_scratch_bytes()


def ra_zigzag_permute(src, n_blocks: int, inverse: bool = False, dst=None, stream=None):
    """Rows of [B, S, H, D] between original and zigzag block order (bit-exact)."""
    B, S, H, D = src.shape
    if dst is None:
        dst = torch.empty_like(src)
    _check(_lib.ra_zigzag_permute(_ptr(src), _ptr(dst), B, S, H, D, src.element_size(), n_blocks,
                                  int(bool(inverse)), _stream(stream)), "ra_zigzag_permute")
    return dst


def ra_get_device_status(stream=None) -> int:
    """Reads and clears the device status word (synchronises the stream)."""
    return _lib.ra_get_device_status(_stream(stream))


def ra_decode_workspace(B, Tq, Skv, Hq, Hkv, D, n_splits=0) -> int:
    n = _lib.ra_decode_workspace(B, Tq, Skv, Hq, Hkv, D, n_splits)
    if n == ctypes.c_size_t(-1).value:
        raise RAError(RA_ERR_INVALID_ARG, "ra_decode_workspace")
    return n


def ra_decode_splits(B, Tq, Skv, Hq, Hkv, D, n_splits=0) -> int:
    n = _lib.ra_decode_splits(B, Tq, Skv, Hq, Hkv, D, n_splits)
    if n < 0:
        raise RAError(RA_ERR_INVALID_ARG, "ra_decode_splits")
    return n


def ra_decode_attention(q, k, v, causal: bool = True, n_splits: int = 0, out=None, lse=None, out_dtype=None,
                        workspace=None, stream=None):
    """Decode attention of q [B, Tq, Hq, D] (the last Tq tokens) over the
    cache k, v [B, Skv, Hkv, D], bf16, in n_splits chunks (0 = chosen to fill
    the GPU).  Returns (out [B, Tq, Hq, D], lse [B, Tq, Hq] fp32)."""
    B, Tq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    for t in (q, k, v):
        if not t.is_contiguous():
            raise RAError(RA_ERR_INVALID_ARG, "ra_decode_attention (tensors must be contiguous)")
    odt = out_dtype or (out.dtype if out is not None else torch.float32)
    if out is None:
        out = torch.empty((B, Tq, Hq, D), dtype=odt, device=q.device)
    if lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    need = ra_decode_workspace(B, Tq, Skv, Hq, Hkv, D, n_splits)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check(_lib.ra_decode_attention(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, Tq, Skv, Hq, Hkv, D,
                                    1 if causal else 0, n_splits, _ptr(out), _dtype_code(out.dtype), _ptr(lse),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "ra_decode_attention")
    return out, lse

