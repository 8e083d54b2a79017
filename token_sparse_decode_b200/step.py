"""Decode steps composed from the C-ABI entry points (device buffers held by torch).

``SparseDecodeStep``: the head-role-split step in one ``aoh_decode_step`` call.  KV
heads with role SPARSE run the importance scan over their dominant chunks, the
top-N_fac select and focused attention; DENSE / STREAM heads attend over the whole
cache or the sink + window.  All write into one fp32 output.

``SharedIndexStep``: the shared-index cross-decoder stack.  The indexer scores
every cached token with the full-dimension q.k, takes one top-k and every layer
attends over that index.  By default that is one ``aoh_shared_index_step`` call
(the library runs it as one cluster kernel or as scan, select and gather kernels);
``fused=False`` makes the three public calls instead (``aoh_tip_score`` with every
chunk, ``aoh_topk_select``, ``aoh_shared_index_decode``).

Every call is asynchronous on the current torch stream; nothing is computed in
Python.
"""

from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import binding as B


class SparseDecodeStep:
    def __init__(self, k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, max_len: int, total_tokens: int,
                 n_q_heads: int, roles: Sequence[int], scale: float, idom: Optional[torch.Tensor] = None,
                 n_fac: int = 0, n_fac_per_seq: Optional[torch.Tensor] = None, n_fac_cap: int = 0,
                 sink: int = 0, window: int = 0, pack_dominant: bool = True):
        self.dev = k.device
        self.k, self.v, self.offsets = k, v, offsets
        self.roles = [int(r) for r in roles]
        self.n_q_heads = n_q_heads
        self.scale = float(scale)
        self.sink, self.window = int(sink), int(window)
        self.has_sparse = any(r == B.ROLE_SPARSE for r in self.roles)
        self.has_stream = any(r != B.ROLE_SPARSE for r in self.roles)
        self.idom = idom
        self.n_dom = 0 if idom is None else idom.shape[1]
        self.n_fac, self.n_fac_per_seq, self.n_fac_cap = int(n_fac), n_fac_per_seq, int(n_fac_cap)
        batch = offsets.numel() - 1
        d = k.shape[2]
        self.k_dom = None
        if self.has_sparse and pack_dominant:
            cols = B.k_dom_cols(self.n_dom)
            self.k_dom = torch.empty((k.shape[1], total_tokens, cols), dtype=torch.bfloat16, device=self.dev)
            kv0 = B.make_kv(k, v, offsets, max_len, total_tokens)
            B.pack_dominant(kv0, idom, self.n_dom, self.k_dom)
        self.kv = B.make_kv(k, v, offsets, max_len, total_tokens, self.k_dom)
        self.n_fac_cap = max(self.n_fac_cap, 1)
        self.idx = self.count = None
        if self.has_sparse:
            self.idx = torch.empty((batch, k.shape[1], self.n_fac_cap), dtype=torch.int32, device=self.dev)
            self.count = torch.empty((batch, k.shape[1]), dtype=torch.int32, device=self.dev)
        self.ws = B.workspace(B.decode_step_workspace_size(self.kv, n_q_heads, self.n_fac_cap, self.roles, self.sink,
                                                           self.window), self.dev)
        self.out = torch.zeros((batch, n_q_heads, d), dtype=torch.float32, device=self.dev)

    def __call__(self, q: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Every head of the step in one ``aoh_decode_step`` call (one launch when the rows allow)."""
        out = self.out if out is None else out
        B.decode_step(q, self.kv, self.idom, self.n_dom, self.n_fac, self.n_fac_per_seq, self.n_fac_cap, self.roles,
                      self.sink, self.window, self.scale, out, self.ws, self.idx, self.count)
        return out

    def run_host(self, q_host: torch.Tensor, out_host: torch.Tensor, q_dev: torch.Tensor) -> None:
        """End-to-end call with host buffers: H2D of q, the step, D2H of the output (async)."""
        q_dev.copy_(q_host, non_blocking=True)
        self(q_dev)
        out_host.copy_(self.out, non_blocking=True)


class SharedIndexStep:
    """fused=True: one ``aoh_shared_index_step`` call; False: score, select, decode as three calls."""

    def __init__(self, k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, max_len: int, total_tokens: int,
                 n_layers: int, n_q_heads: int, topk: int, scale: float, fused: bool = True):
        self.fused = fused
        self.dev = k.device
        self.k, self.v, self.offsets = k, v, offsets
        self.kv = B.make_kv(k, v, offsets, max_len, total_tokens)
        Hkv, d = k.shape[1], k.shape[2]
        batch = offsets.numel() - 1
        self.n_layers, self.n_q_heads, self.topk, self.scale = n_layers, n_q_heads, int(topk), float(scale)
        self.all_chunks = torch.arange(d // 2, dtype=torch.int32, device=self.dev).repeat(Hkv, 1).contiguous()
        self.idx = torch.empty((batch, Hkv, self.topk), dtype=torch.int32, device=self.dev)
        self.count = torch.empty((batch, Hkv), dtype=torch.int32, device=self.dev)
        if fused:  # the step's workspace holds its own scores
            self.scores = self.ws = None
            self.ws_step = B.workspace(B.shared_index_step_workspace_size(self.kv, n_layers, n_q_heads, self.topk),
                                       self.dev)
        else:
            self.scores = torch.empty((Hkv, max(total_tokens, 1)), dtype=torch.float32, device=self.dev)
            self.ws = B.workspace(B.shared_index_decode_workspace_size(self.kv, n_layers, n_q_heads, self.topk),
                                  self.dev)
            self.ws_select = B.workspace(B.topk_select_workspace_size(self.kv), self.dev)
            self.ws_step = None
        self.out = torch.zeros((n_layers, batch, n_q_heads, d), dtype=torch.float32, device=self.dev)

    def index(self, q_index: torch.Tensor) -> None:
        if self.scores is None:
            raise RuntimeError("SharedIndexStep.index needs fused=False (the fused step keeps its scores inside)")
        B.tip_score(q_index, self.kv, self.all_chunks, self.all_chunks.shape[1], self.scores)
        B.topk_select(self.scores, self.kv, self.topk, None, self.topk, self.idx, self.count, self.ws_select)

    def __call__(self, q_index: torch.Tensor, q_layers: torch.Tensor) -> torch.Tensor:
        if self.fused:
            B.shared_index_step(q_index, q_layers, self.kv, self.topk, self.idx, self.count, self.scale, self.out,
                                self.ws_step)
            return self.out
        self.index(q_index)
        B.shared_index_decode(q_layers, self.kv, self.idx, self.count, self.topk, self.scale, self.out, self.ws)
        return self.out


class AppendDecodeStep:
    """Decode steps that first append their token (``aoh_kv_append``), then attend.

    The AoH deployment of the head roles: SPARSE and DENSE KV heads keep their whole
    history in a linear cache with a fixed capacity per sequence; STREAM heads keep only
    a ring of ``sink + window`` slots per sequence.  Each cache holds only its own heads
    (head slots), so a streaming head costs sink + window rows, not its sequence length.
    ``lengths`` (device int32 [B]) is the one position counter both caches share.

    One call: rotate the new q and k to position lengths[b], write the K / V rows (and the
    packed dominant row of each linear-cache head), lengths += 1; then the SPARSE heads'
    importance scan / top-N_fac / focused attention and the DENSE heads' full attention on
    the linear cache, and the STREAM heads' sink + window attention on the ring.  The
    query attends over positions 0 .. p, its own token included.
    """

    def __init__(self, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, theta: float,
                 roles: Sequence[int], capacity: Sequence[int], sink: int, window: int, scale: float,
                 idom: Optional[torch.Tensor] = None, n_fac: int = 0, device="cuda"):
        self.dev = torch.device(device)
        self.B, self.Hq, self.Hkv, self.d = batch, n_q_heads, n_kv_heads, head_dim
        self.theta, self.scale = float(theta), float(scale)
        self.roles = [int(r) for r in roles]
        self.sink, self.window = int(sink), int(window)
        self.idom = idom
        self.n_dom = 0 if idom is None else idom.shape[1]
        self.n_fac = int(n_fac)
        lin = [g for g in range(n_kv_heads) if self.roles[g] != B.ROLE_STREAM]
        rng = [g for g in range(n_kv_heads) if self.roles[g] == B.ROLE_STREAM]
        self.lin_slot = [lin.index(g) if g in lin else B.NO_SLOT for g in range(n_kv_heads)]
        self.ring_slot = [rng.index(g) if g in rng else B.NO_SLOT for g in range(n_kv_heads)]
        self.has_sparse = any(r == B.ROLE_SPARSE for r in self.roles)
        self.has_dense = any(r == B.ROLE_DENSE for r in self.roles)
        self.has_stream = bool(rng)
        cap = [int(c) for c in capacity]
        assert len(cap) == batch
        self.capacity = cap
        offs = [0]
        for c in cap:
            offs.append(offs[-1] + c)
        self.offsets = torch.tensor(offs, dtype=torch.int32, device=self.dev)
        self.lengths = torch.zeros(batch, dtype=torch.int32, device=self.dev)
        T, max_len = offs[-1], max(cap) if cap else 0
        self.k = torch.zeros((max(T, 1), max(len(lin), 1), head_dim), dtype=torch.bfloat16, device=self.dev)
        self.v = torch.zeros_like(self.k)
        self.k_dom = None
        if self.has_sparse:
            assert idom is not None and idom.shape[0] == n_kv_heads
            self.k_dom = torch.zeros((max(len(lin), 1), max(T, 1), B.k_dom_cols(self.n_dom)), dtype=torch.bfloat16,
                                     device=self.dev)
        self.kv = None
        if lin:
            self.kv = B.make_kv(self.k, self.v, self.offsets, max_len, T, self.k_dom, self.lengths, self.lin_slot,
                                n_kv_heads)
        self.ring = None
        if rng:
            slots = self.sink + self.window
            self.ring_offsets = torch.arange(0, (batch + 1) * slots, slots, dtype=torch.int32, device=self.dev)
            self.rk = torch.zeros((max(batch * slots, 1), len(rng), head_dim), dtype=torch.bfloat16, device=self.dev)
            self.rv = torch.zeros_like(self.rk)
            self.ring = B.make_kv(self.rk, self.rv, self.ring_offsets, max_len, batch * slots, None, self.lengths,
                                  self.ring_slot, n_kv_heads, ring=(self.sink, self.window))
        self.q_rot = torch.zeros((batch, n_q_heads, head_dim), dtype=torch.bfloat16, device=self.dev)
        self.out = torch.zeros((batch, n_q_heads, head_dim), dtype=torch.float32, device=self.dev)
        self.idx = self.count = self.ws_sparse = self.ws_dense = self.ws_ring = None
        if self.has_sparse:
            self.idx = torch.empty((batch, n_kv_heads, max(self.n_fac, 1)), dtype=torch.int32, device=self.dev)
            self.count = torch.empty((batch, n_kv_heads), dtype=torch.int32, device=self.dev)
            self.ws_sparse = B.workspace(B.sparse_decode_workspace_size(self.kv, n_q_heads, max(self.n_fac, 1)),
                                         self.dev)
        if self.has_dense:
            self.ws_dense = B.workspace(B.stream_decode_workspace_size(self.kv, n_q_heads, self.roles, 0, 0), self.dev)
        if self.has_stream:
            self.ws_ring = B.workspace(B.stream_decode_workspace_size(self.ring, n_q_heads, self.roles, self.sink,
                                                                      self.window), self.dev)

    def append(self, q_new: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor) -> None:
        B.kv_append(q_new, k_new, v_new, self.theta, self.kv, self.ring, self.idom, self.n_dom, self.lengths,
                    self.q_rot)

    def decode(self) -> torch.Tensor:
        if self.has_sparse:
            B.sparse_decode(self.q_rot, self.kv, self.idom, self.n_dom, self.n_fac, None, max(self.n_fac, 1),
                            self.roles, self.scale, self.out, self.ws_sparse, self.idx, self.count)
        if self.has_dense:
            B.stream_decode(self.q_rot, self.kv, self.roles, 0, 0, self.scale, self.out, self.ws_dense)
        if self.has_stream:
            B.stream_decode(self.q_rot, self.ring, self.roles, self.sink, self.window, self.scale, self.out,
                            self.ws_ring)
        return self.out

    def __call__(self, q_new: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor) -> torch.Tensor:
        self.append(q_new, k_new, v_new)
        return self.decode()


class OffloadDecodeStep:
    """FASA-M decode step: V and the non-dominant key dims in pinned host memory.

    Built from a device cache: the dominant columns are packed into device memory
    (``aoh_pack_dominant``) and the rest of K and all of V are written to pinned host
    buffers (``aoh_offload_split``); the device K / V are not kept.  A call is one
    ``aoh_offload_decode``: scan and select on the GPU, the selected rows across the host
    link, focused attention.  Every KV head is SPARSE.
    """

    def __init__(self, k: torch.Tensor, v: torch.Tensor, offsets: torch.Tensor, max_len: int, total_tokens: int,
                 n_q_heads: int, idom: torch.Tensor, scale: float, n_fac: int = 0,
                 n_fac_per_seq: Optional[torch.Tensor] = None, n_fac_cap: int = 0,
                 lengths: Optional[torch.Tensor] = None):
        self.dev = k.device
        Hkv, d = k.shape[1], k.shape[2]
        self.idom, self.n_dom = idom, idom.shape[1]
        self.scale, self.n_fac, self.n_fac_per_seq, self.n_fac_cap = float(scale), int(n_fac), n_fac_per_seq, int(n_fac_cap)
        kv = B.make_kv(k, v, offsets, max_len, total_tokens, lengths=lengths)
        self.k_dom = torch.empty((Hkv, max(total_tokens, 1), B.k_dom_cols(self.n_dom)), dtype=torch.bfloat16,
                                 device=self.dev)
        B.pack_dominant(kv, idom, self.n_dom, self.k_dom)
        self.k_rest = torch.empty((Hkv, max(total_tokens, 1), B.rest_cols(d, self.n_dom)), dtype=torch.bfloat16,
                                  pin_memory=True)
        self.v_host = torch.empty((Hkv, max(total_tokens, 1), d), dtype=torch.bfloat16, pin_memory=True)
        B.offload_split(kv, idom, self.n_dom, self.k_rest, self.v_host)
        torch.cuda.current_stream().synchronize()  # the host parts are complete before k, v may go
        self.oc = B.make_offload(offsets, max_len, total_tokens, Hkv, d, self.k_dom, self.k_rest, self.v_host, lengths)
        batch = offsets.numel() - 1
        self.idx = torch.empty((batch, Hkv, self.n_fac_cap), dtype=torch.int32, device=self.dev)
        self.count = torch.empty((batch, Hkv), dtype=torch.int32, device=self.dev)
        self.ws = B.workspace(B.offload_decode_workspace_size(self.oc, n_q_heads, self.n_fac_cap), self.dev)
        self.out = torch.zeros((batch, n_q_heads, d), dtype=torch.float32, device=self.dev)

    def link_bytes_per_step(self) -> int:
        """Bytes that cross the host link per step: the selected rows' rest-of-K and V."""
        n = self.count.to(torch.int64).sum().item()
        return int(n) * 2 * (self.k_rest.shape[-1] + self.v_host.shape[-1])

    def __call__(self, q: torch.Tensor) -> torch.Tensor:
        B.offload_decode(q, self.oc, self.idom, self.n_dom, self.n_fac, self.n_fac_per_seq, self.n_fac_cap,
                         self.scale, self.out, self.ws, self.idx, self.count)
        return self.out
