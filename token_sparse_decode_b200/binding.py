"""ctypes binding of libaoh.so: argument marshalling only.

Every entry point takes torch CUDA tensors, turns them into raw device pointers
and sizes, calls the C function of the same name on the current torch stream and
raises AohError on a non-zero status.  No arithmetic of the decode step happens
here; if the library is missing the import fails (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaoh.so")

ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM = 0, 1, 2
STATUS = {0: "AOH_OK", 1: "AOH_ERR_INVALID_ARG", 2: "AOH_ERR_UNSUPPORTED", 3: "AOH_ERR_ALIGNMENT",
          4: "AOH_ERR_WORKSPACE", 5: "AOH_ERR_CUDA", 6: "AOH_ERR_DEVICE_CHECK"}

EXPORTS = (
    "aoh_status_string", "aoh_version", "aoh_last_cuda_error", "aoh_device_check", "aoh_pack_dominant", "aoh_tip_score",
    "aoh_topk_select", "aoh_sparse_decode", "aoh_sparse_decode_workspace_size", "aoh_stream_decode",
    "aoh_stream_decode_workspace_size", "aoh_shared_index_decode", "aoh_shared_index_decode_workspace_size",
    "aoh_shared_index_step", "aoh_shared_index_step_workspace_size", "aoh_stream_decode_noalloc",
    "aoh_launch_counts", "aoh_record_launch_events", "aoh_kv_append", "aoh_head_classify",
    "aoh_head_classify_workspace_size", "aoh_topk_select_workspace_size", "aoh_decode_step",
    "aoh_decode_step_workspace_size", "aoh_offload_split", "aoh_offload_decode", "aoh_offload_decode_workspace_size",
)
NO_SLOT = 255  # head_slot entry of a KV head a cache does not store

# aoh_kernel_kind order
KERNELS = ("tip_score_kernel", "select_hist_kernel", "sparse_row_kernel", "flash_gather_kernel",
           "pack_dominant_kernel", "kv_append_kernel", "gram_kernel", "gram_reduce_kernel", "spectrum_kernel",
           "group_roles_kernel", "offload_stage_kernel", "offload_split_kernel", "select_chunk_kernel",
           "select_write_kernel", "select_cluster_kernel",
           "select_resolve_kernel", "flash_merge_kernel")


class AohError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        extra = f" (cudaError {cuda_error})" if cuda_error else ""
        super().__init__(f"{fn}: {STATUS.get(status, status)}{extra}")


class KVCache(ctypes.Structure):
    """Mirror of ``aoh_kv_cache`` (include/aoh.h)."""

    _fields_ = [
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("offsets", ctypes.c_void_p),
        ("batch", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("max_len", ctypes.c_int32), ("total_tokens", ctypes.c_int64), ("stride_tok", ctypes.c_int64),
        ("stride_head", ctypes.c_int64), ("k_dom", ctypes.c_void_p), ("k_dom_cols", ctypes.c_int32),
        ("lengths", ctypes.c_void_p), ("head_slot", ctypes.c_void_p), ("ring_sink", ctypes.c_int32),
        ("ring_window", ctypes.c_int32),
    ]


class OffloadCache(ctypes.Structure):
    """Mirror of ``aoh_offload_cache`` (include/aoh.h)."""

    _fields_ = [
        ("offsets", ctypes.c_void_p), ("lengths", ctypes.c_void_p), ("batch", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("max_len", ctypes.c_int32),
        ("total_tokens", ctypes.c_int64), ("k_dom", ctypes.c_void_p), ("k_dom_cols", ctypes.c_int32),
        ("rest_cols", ctypes.c_int32), ("k_rest", ctypes.c_void_p), ("v", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libaoh.so once (after torch, so that it binds to torch's CUDA runtime)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built: run `python -m token_sparse_decode_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        KVP = ctypes.POINTER(KVCache)
        sig = {
            "aoh_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "aoh_version": (I32, []),
            "aoh_last_cuda_error": (I32, []),
            "aoh_device_check": (ctypes.c_int, [P, P]),
            "aoh_launch_counts": (I32, [P, I32]),
            "aoh_record_launch_events": (None, [P, P, I32]),
            "aoh_pack_dominant": (ctypes.c_int, [KVP, P, I32, P, I32, P]),
            "aoh_tip_score": (ctypes.c_int, [P, I32, KVP, P, I32, P, P]),
            "aoh_topk_select": (ctypes.c_int, [P, KVP, I32, P, I32, P, P, P, SZ, P]),
            "aoh_topk_select_workspace_size": (SZ, [KVP]),
            "aoh_decode_step": (ctypes.c_int, [P, I32, KVP, P, I32, I32, P, I32, P, I32, I32, F32, P, P, P, P, SZ, P]),
            "aoh_decode_step_workspace_size": (SZ, [KVP, I32, I32, P, I32, I32]),
            "aoh_sparse_decode": (ctypes.c_int, [P, I32, KVP, P, I32, I32, P, I32, P, F32, P, P, P, P, SZ, P]),
            "aoh_sparse_decode_workspace_size": (SZ, [KVP, I32, I32]),
            "aoh_stream_decode": (ctypes.c_int, [P, I32, KVP, P, I32, I32, F32, P, P, SZ, P]),
            "aoh_stream_decode_workspace_size": (SZ, [KVP, I32, P, I32, I32]),
            "aoh_shared_index_decode": (ctypes.c_int, [P, I32, I32, KVP, P, P, I32, F32, P, P, SZ, P]),
            "aoh_shared_index_decode_workspace_size": (SZ, [KVP, I32, I32, I32]),
            "aoh_shared_index_step": (ctypes.c_int, [P, P, I32, I32, KVP, I32, P, P, F32, P, P, SZ, P]),
            "aoh_shared_index_step_workspace_size": (SZ, [KVP, I32, I32, I32]),
            "aoh_stream_decode_noalloc": (ctypes.c_int, [P, I32, KVP, P, I32, I32, F32, P, P]),
            "aoh_kv_append": (ctypes.c_int, [P, I32, P, P, ctypes.c_double, KVP, KVP, P, I32, P, P, P]),
            "aoh_head_classify": (ctypes.c_int, [P, P, I32, I32, I32, I32, I32, P, P, P, P, SZ, P]),
            "aoh_head_classify_workspace_size": (SZ, [I32, I32, I32, I32]),
            "aoh_offload_split": (ctypes.c_int, [KVP, P, I32, P, I32, P, P]),
            "aoh_offload_decode": (ctypes.c_int, [P, I32, ctypes.POINTER(OffloadCache), P, I32, I32, P, I32, F32, P, P, P,
                                                  P, SZ, P]),
            "aoh_offload_decode_workspace_size": (SZ, [ctypes.POINTER(OffloadCache), I32, I32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise AohError(fn, status, lib().aoh_last_cuda_error() if status == 5 else 0)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _host_u8(arr) -> Optional[ctypes.Array]:
    if arr is None:
        return None
    vals = [int(x) for x in (arr.tolist() if hasattr(arr, "tolist") else arr)]
    return (ctypes.c_uint8 * len(vals))(*vals)


def make_kv(k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, max_len: int, total_tokens: int,
            k_dom: Optional[torch.Tensor] = None, lengths: Optional[torch.Tensor] = None, head_slot=None,
            n_kv_heads: Optional[int] = None, ring: Optional[tuple] = None) -> KVCache:
    """Describe a cache held in torch tensors k, v of shape [T, slots, d] (bf16, last dim contiguous).

    lengths: device int32 [B] (positions held per sequence) or None (sequences fill their regions);
    head_slot: per KV head its slot in k / v (NO_SLOT: not stored here), or None (identity, slots = heads);
    n_kv_heads: the model's KV heads (default: k.shape[1]); ring: (sink, window) for a ring layout.
    """
    assert k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16 and k.is_cuda and v.is_cuda
    assert k.shape == v.shape and k.stride() == v.stride() and k.stride(2) == 1
    assert offsets.dtype == torch.int32 and offsets.is_cuda
    assert lengths is None or (lengths.dtype == torch.int32 and lengths.is_cuda)
    kv = KVCache()
    slots = None if head_slot is None else (ctypes.c_uint8 * len(head_slot))(*[int(x) for x in head_slot])
    kv._keep = (k, v, offsets, k_dom, lengths, slots)  # raw pointers: keep their owners alive with the descriptor
    kv.k, kv.v, kv.offsets = k.data_ptr(), v.data_ptr(), offsets.data_ptr()
    kv.batch = offsets.numel() - 1
    kv.n_kv_heads = n_kv_heads if n_kv_heads is not None else k.shape[1]
    kv.head_dim = k.shape[2]
    if lengths is not None:
        kv.lengths = lengths.data_ptr()
    if slots is not None:
        assert len(head_slot) == kv.n_kv_heads
        kv.head_slot = ctypes.cast(slots, ctypes.c_void_p).value
    if ring is not None:
        kv.ring_sink, kv.ring_window = int(ring[0]), int(ring[1])
    kv.max_len = int(max_len)
    kv.total_tokens = int(total_tokens)
    kv.stride_tok = k.stride(0)
    kv.stride_head = k.stride(1)
    if k_dom is not None:
        assert k_dom.dtype == torch.bfloat16 and k_dom.is_cuda and k_dom.is_contiguous()
        kv.k_dom = k_dom.data_ptr()
        kv.k_dom_cols = k_dom.shape[-1]
    return kv


def k_dom_cols(n_dom: int) -> int:
    """Row length of the packed dominant-column copy: 2*n_dom rounded up to 16 * 2^j elements."""
    c = 16
    while c < 2 * n_dom:
        c *= 2
    return c


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled device buffer (the allocator gives >= 512-byte alignment)."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------- entry points

def launch_counts() -> dict:
    """Kernel launches made through the library so far, by kernel name (host counters)."""
    n = len(KERNELS)
    buf = (ctypes.c_int64 * n)()
    kinds = lib().aoh_launch_counts(ctypes.cast(buf, ctypes.c_void_p), n)
    if kinds != n:
        raise AohError("aoh_launch_counts", 1)
    return {name: int(buf[i]) for i, name in enumerate(KERNELS)}


def timed_launches(fn, events=None, max_launches: int = 8):
    """Run fn() (one library call) with launch-event recording armed.

    Returns [(kernel name, start event, end event)] for the kernels fn() launched, in
    launch order; the events are recorded on each launch's stream, so elapsed_time of a
    pair (after a synchronize) is that kernel's device time.  `events` (max_launches + 1
    timing events) may be passed in to be reused.
    """
    n = max_launches + 1
    evs = events if events is not None else [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    if len(evs) != n:
        raise ValueError("timed_launches: need max_launches + 1 events")
    for ev in evs:
        if not ev.cuda_event:  # created on first record
            ev.record()
    handles = (ctypes.c_void_p * n)(*[ev.cuda_event for ev in evs])
    kinds = (ctypes.c_int32 * max_launches)(*([-1] * max_launches))
    L = lib()
    L.aoh_record_launch_events(ctypes.cast(handles, ctypes.c_void_p), ctypes.cast(kinds, ctypes.c_void_p), n)
    try:
        fn()
    finally:
        L.aoh_record_launch_events(None, None, 0)
    out = []
    for i in range(max_launches):
        if kinds[i] < 0:
            break
        out.append((KERNELS[kinds[i]], evs[i], evs[i + 1]))
    return out


def device_check(stream=None):
    detail = (ctypes.c_int32 * 4)()
    st = lib().aoh_device_check(_stream(stream), ctypes.cast(detail, ctypes.c_void_p))
    return st, list(detail)


def pack_dominant(kv: KVCache, idom: torch.Tensor, n_dom: int, k_dom: torch.Tensor, stream=None) -> None:
    _check("aoh_pack_dominant", lib().aoh_pack_dominant(ctypes.byref(kv), _ptr(idom), n_dom, _ptr(k_dom),
                                                         k_dom.shape[-1], _stream(stream)))


def tip_score(q: torch.Tensor, kv: KVCache, idom: torch.Tensor, n_dom: int, scores: torch.Tensor,
              stream=None) -> None:
    _check("aoh_tip_score", lib().aoh_tip_score(_ptr(q), q.shape[-2], ctypes.byref(kv), _ptr(idom), n_dom,
                                                 _ptr(scores), _stream(stream)))


def topk_select_workspace_size(kv: KVCache) -> int:
    return int(lib().aoh_topk_select_workspace_size(ctypes.byref(kv)))


def topk_select(scores: torch.Tensor, kv: KVCache, n_fac: int, n_fac_per_seq: Optional[torch.Tensor],
                n_fac_cap: int, idx: torch.Tensor, count: torch.Tensor, ws: Optional[torch.Tensor] = None,
                stream=None) -> None:
    """aoh_topk_select; without `ws` a zero-filled workspace of the required size is made here."""
    if ws is None:
        ws = workspace(topk_select_workspace_size(kv), scores.device)
    _check("aoh_topk_select", lib().aoh_topk_select(_ptr(scores), ctypes.byref(kv), n_fac, _ptr(n_fac_per_seq),
                                                     n_fac_cap, _ptr(idx), _ptr(count), _ptr(ws), ws.numel(),
                                                     _stream(stream)))


def sparse_decode_workspace_size(kv: KVCache, n_q_heads: int, n_fac_cap: int) -> int:
    return int(lib().aoh_sparse_decode_workspace_size(ctypes.byref(kv), n_q_heads, n_fac_cap))


def sparse_decode(q: torch.Tensor, kv: KVCache, idom: torch.Tensor, n_dom: int, n_fac: int,
                  n_fac_per_seq: Optional[torch.Tensor], n_fac_cap: int, roles, scale: float,
                  out: torch.Tensor, ws: torch.Tensor, idx_out: Optional[torch.Tensor] = None,
                  count_out: Optional[torch.Tensor] = None, stream=None) -> None:
    r = _host_u8(roles)
    _check("aoh_sparse_decode", lib().aoh_sparse_decode(
        _ptr(q), q.shape[-2], ctypes.byref(kv), _ptr(idom), n_dom, n_fac, _ptr(n_fac_per_seq), n_fac_cap,
        None if r is None else ctypes.cast(r, ctypes.c_void_p), float(scale), _ptr(out), _ptr(idx_out),
        _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)))


def stream_decode_workspace_size(kv: KVCache, n_q_heads: int, roles, sink: int, window: int) -> int:
    r = _host_u8(roles)
    return int(lib().aoh_stream_decode_workspace_size(ctypes.byref(kv), n_q_heads,
                                                      ctypes.cast(r, ctypes.c_void_p), sink, window))


def stream_decode(q: torch.Tensor, kv: KVCache, roles, sink: int, window: int, scale: float,
                  out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    r = _host_u8(roles)
    _check("aoh_stream_decode", lib().aoh_stream_decode(
        _ptr(q), q.shape[-2], ctypes.byref(kv), ctypes.cast(r, ctypes.c_void_p), sink, window, float(scale),
        _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def decode_step_workspace_size(kv: KVCache, n_q_heads: int, n_fac_cap: int, roles, sink: int, window: int) -> int:
    r = _host_u8(roles)
    return int(lib().aoh_decode_step_workspace_size(ctypes.byref(kv), n_q_heads, n_fac_cap,
                                                    None if r is None else ctypes.cast(r, ctypes.c_void_p), sink,
                                                    window))


def decode_step(q: torch.Tensor, kv: KVCache, idom: Optional[torch.Tensor], n_dom: int, n_fac: int,
                n_fac_per_seq: Optional[torch.Tensor], n_fac_cap: int, roles, sink: int, window: int, scale: float,
                out: torch.Tensor, ws: torch.Tensor, idx_out: Optional[torch.Tensor] = None,
                count_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """Every head of the step, by role (aoh_decode_step)."""
    r = _host_u8(roles)
    _check("aoh_decode_step", lib().aoh_decode_step(
        _ptr(q), q.shape[-2], ctypes.byref(kv), _ptr(idom), n_dom, n_fac, _ptr(n_fac_per_seq), n_fac_cap,
        None if r is None else ctypes.cast(r, ctypes.c_void_p), sink, window, float(scale), _ptr(out), _ptr(idx_out),
        _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)))


def shared_index_decode_workspace_size(kv: KVCache, n_layers: int, n_q_heads: int, n_fac_cap: int) -> int:
    return int(lib().aoh_shared_index_decode_workspace_size(ctypes.byref(kv), n_layers, n_q_heads, n_fac_cap))


def shared_index_decode(q_layers: torch.Tensor, kv: KVCache, idx: torch.Tensor, count: torch.Tensor,
                        n_fac_cap: int, scale: float, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check("aoh_shared_index_decode", lib().aoh_shared_index_decode(
        _ptr(q_layers), q_layers.shape[0], q_layers.shape[-2], ctypes.byref(kv), _ptr(idx), _ptr(count),
        n_fac_cap, float(scale), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def shared_index_step_workspace_size(kv: KVCache, n_layers: int, n_q_heads: int, topk: int) -> int:
    return int(lib().aoh_shared_index_step_workspace_size(ctypes.byref(kv), n_layers, n_q_heads, topk))


def shared_index_step(q_index: torch.Tensor, q_layers: torch.Tensor, kv: KVCache, topk: int, idx: torch.Tensor,
                      count: torch.Tensor, scale: float, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    _check("aoh_shared_index_step", lib().aoh_shared_index_step(
        _ptr(q_index), _ptr(q_layers), q_layers.shape[0], q_layers.shape[-2], ctypes.byref(kv), topk, _ptr(idx),
        _ptr(count), float(scale), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def stream_decode_noalloc(q: torch.Tensor, kv: KVCache, roles, sink: int, window: int, scale: float,
                          out: torch.Tensor, stream=None) -> None:
    """aoh_stream_decode with the library's own static scratch (no workspace argument)."""
    r = _host_u8(roles)
    _check("aoh_stream_decode_noalloc", lib().aoh_stream_decode_noalloc(
        _ptr(q), q.shape[-2], ctypes.byref(kv), ctypes.cast(r, ctypes.c_void_p), sink, window, float(scale),
        _ptr(out), _stream(stream)))


def kv_append(q_new: Optional[torch.Tensor], k_new: torch.Tensor, v_new: torch.Tensor, theta: float,
              kv: Optional[KVCache], ring: Optional[KVCache], idom: Optional[torch.Tensor], n_dom: int,
              lengths: torch.Tensor, q_out: Optional[torch.Tensor], stream=None) -> None:
    """Rotate and append every sequence's decoded token (aoh_kv_append); lengths[b] += 1."""
    _check("aoh_kv_append", lib().aoh_kv_append(
        _ptr(q_new), 0 if q_new is None else q_new.shape[-2], _ptr(k_new), _ptr(v_new), float(theta),
        None if kv is None else ctypes.byref(kv), None if ring is None else ctypes.byref(ring), _ptr(idom),
        int(n_dom), _ptr(lengths), _ptr(q_out), _stream(stream)))


def head_classify_workspace_size(d_model: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> int:
    return int(lib().aoh_head_classify_workspace_size(d_model, n_q_heads, n_kv_heads, head_dim))


def head_classify(w_q: torch.Tensor, w_k: torch.Tensor, n_q_heads: int, n_kv_heads: int, head_dim: int,
                  n_retrieval: int, er_heads: torch.Tensor, er_groups: torch.Tensor, roles: torch.Tensor,
                  ws: torch.Tensor, stream=None) -> None:
    """AoH head classification from bf16 projection weights w_q [Hq*d, d_model], w_k [Hkv*d, d_model]."""
    assert w_q.dtype == torch.bfloat16 and w_k.dtype == torch.bfloat16 and w_q.is_contiguous() and w_k.is_contiguous()
    assert er_heads.dtype == torch.float64 and er_groups.dtype == torch.float64 and roles.dtype == torch.uint8
    _check("aoh_head_classify", lib().aoh_head_classify(
        _ptr(w_q), _ptr(w_k), w_q.shape[1], n_q_heads, n_kv_heads, head_dim, n_retrieval, _ptr(er_heads),
        _ptr(er_groups), _ptr(roles), _ptr(ws), ws.numel(), _stream(stream)))


def rest_cols(head_dim: int, n_dom: int) -> int:
    """Row length of the host copy of the non-dominant key dims: d - 2 n_dom rounded up to 8."""
    return (head_dim - 2 * n_dom + 7) // 8 * 8


def make_offload(offsets: torch.Tensor, max_len: int, total_tokens: int, n_kv_heads: int, head_dim: int,
                 k_dom: torch.Tensor, k_rest: torch.Tensor, v: torch.Tensor,
                 lengths: Optional[torch.Tensor] = None) -> OffloadCache:
    """Describe a FASA-M cache: k_dom on the device, k_rest and v in pinned host memory."""
    assert k_dom.is_cuda and not k_rest.is_cuda and not v.is_cuda
    assert k_rest.is_pinned() and v.is_pinned(), "host parts must be pinned"
    oc = OffloadCache()
    oc._keep = (offsets, k_dom, k_rest, v, lengths)
    oc.offsets = offsets.data_ptr()
    if lengths is not None:
        oc.lengths = lengths.data_ptr()
    oc.batch = offsets.numel() - 1
    oc.n_kv_heads, oc.head_dim, oc.max_len, oc.total_tokens = n_kv_heads, head_dim, int(max_len), int(total_tokens)
    oc.k_dom, oc.k_dom_cols = k_dom.data_ptr(), k_dom.shape[-1]
    oc.k_rest, oc.rest_cols = k_rest.data_ptr(), k_rest.shape[-1]
    oc.v = v.data_ptr()
    return oc


def offload_split(kv: KVCache, idom: torch.Tensor, n_dom: int, k_rest: torch.Tensor, v_host: torch.Tensor,
                  stream=None) -> None:
    _check("aoh_offload_split", lib().aoh_offload_split(ctypes.byref(kv), _ptr(idom), n_dom, _ptr(k_rest),
                                                         k_rest.shape[-1], _ptr(v_host), _stream(stream)))


def offload_decode_workspace_size(oc: OffloadCache, n_q_heads: int, n_fac_cap: int) -> int:
    return int(lib().aoh_offload_decode_workspace_size(ctypes.byref(oc), n_q_heads, n_fac_cap))


def offload_decode(q: torch.Tensor, oc: OffloadCache, idom: torch.Tensor, n_dom: int, n_fac: int,
                   n_fac_per_seq: Optional[torch.Tensor], n_fac_cap: int, scale: float, out: torch.Tensor,
                   ws: torch.Tensor, idx_out: Optional[torch.Tensor] = None, count_out: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    _check("aoh_offload_decode", lib().aoh_offload_decode(
        _ptr(q), q.shape[-2], ctypes.byref(oc), _ptr(idom), n_dom, n_fac, _ptr(n_fac_per_seq), n_fac_cap,
        float(scale), _ptr(out), _ptr(idx_out), _ptr(count_out), _ptr(ws), ws.numel(), _stream(stream)))
