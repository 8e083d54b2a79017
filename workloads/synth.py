"""Seeded synthetic decode-step inputs (bf16 q, K, V, I_dom, roles, ragged offsets).

Recipe (every draw is keyed by ``(seed, stream tag, indices...)`` through
``numpy.random.SeedSequence`` so that any (sequence, KV head) block can be
regenerated alone):

* K and V rows, and every query head, are i.i.d. standard normal (float32
  draws from PCG64).
* Planted salient keys (the 8B-shaped and the ragged serving workloads): for
  each (sequence b, KV head g), ``ceil(planted_frac * L_b)`` token positions
  are chosen without replacement, and for each of them ``ceil(n_dom / 4)``
  chunks of that head's dominant set are chosen; both coordinates of each such
  chunk are multiplied by ``planted_gain``.  This happens before the rotation
  (it commutes with it, the rotation being linear per chunk).
* Keys are rotated at their absolute positions ``0 .. L_b - 1`` and queries at
  position ``L_b`` (the cache holds every earlier token; the query is the new
  token).  The rotation pairs dims ``(c, c + d/2)`` (rotate-half layout) with
  angle ``p * theta ** (-2c/d)``.  V is not rotated.
* Values are rounded once to bf16 (round to nearest even, from float32).
* The dominant chunk set of each KV head is ``n_dom`` distinct chunk ids drawn
  without replacement from ``0 .. d/2 - 1`` and sorted.
* Ragged lengths are uniform integers in ``[lo, hi]`` (both ends included).
* Head roles: either all SPARSE, an explicit tuple, or ``n_retrieval`` DENSE
  KV groups taken as the first entries of a seeded permutation, the rest
  STREAM.

The rotation here is input synthesis: the decode step consumes keys and
queries that are already rotated and never rotates anything itself.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional, Tuple

import numpy as np
import torch

ROLE_SPARSE = 0  # TIP score -> top-N_fac -> focused attention over the selection
ROLE_DENSE = 1   # retrieval head: attention over the whole cache
ROLE_STREAM = 2  # streaming head: attention over sink tokens + recent window

_TAG_K, _TAG_V, _TAG_Q, _TAG_QL, _TAG_PLANT, _TAG_IDOM, _TAG_ROLE, _TAG_LEN, _TAG_QI = range(1, 10)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *[int(k) for k in key]])))


@dataclass(frozen=True)
class WorkloadSpec:
    """Shape and recipe of one synthetic decode step."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    theta: float
    lengths: Optional[Tuple[int, ...]] = None      # fixed per-sequence cache lengths
    len_range: Optional[Tuple[int, int]] = None    # else drawn uniformly in [lo, hi]
    n_dom: int = 0                                 # |I_dom| per KV head (0: no TIP stage)
    n_fac: int = 0                                 # fixed N_fac ...
    n_fac_div: int = 0                             # ... or N_fac = ceil(L_b / n_fac_div)
    roles: Tuple[int, ...] = ()                    # explicit roles per KV head, or () ...
    n_retrieval: int = -1                          # ... or this many DENSE groups drawn, rest STREAM
    sink: int = 0
    window: int = 0
    planted_frac: float = 0.0
    planted_gain: float = 4.0
    n_layers: int = 0                              # cross-decoder layers sharing one index
    topk_shared: int = 0                           # k of the shared indexer
    seed: int = 1234

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


@dataclass
class Workload:
    spec: WorkloadSpec
    lengths: np.ndarray                 # int64 [B]
    offsets: torch.Tensor               # int32 [B + 1]
    k: torch.Tensor                     # bf16 [T_total, Hkv, d], post-rotation
    v: torch.Tensor                     # bf16 [T_total, Hkv, d]
    q: torch.Tensor                     # bf16 [B, Hq, d] (the indexer's q for the shared-index stack)
    q_layers: Optional[torch.Tensor]    # bf16 [n_layers, B, Hq, d] or None
    idom: Optional[torch.Tensor]        # int32 [Hkv, n_dom], sorted, or None
    roles: torch.Tensor                 # uint8 [Hkv]
    n_fac_per_seq: torch.Tensor         # int32 [B]
    scale: float
    planted: dict = field(default_factory=dict)   # (b, g) -> int64 token positions that were boosted

    @property
    def total_tokens(self) -> int:
        return int(self.lengths.sum())

    @property
    def max_len(self) -> int:
        return int(self.lengths.max()) if len(self.lengths) else 0


# --------------------------------------------------------------------------------------
# rotation used to synthesise post-RoPE inputs (float32 arithmetic, float64 angles)
# --------------------------------------------------------------------------------------

def _angles(n_pos: int, head_dim: int, theta: float, start: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    C = head_dim // 2
    inv_freq = theta ** (-2.0 * np.arange(C, dtype=np.float64) / head_dim)
    ang = np.arange(start, start + n_pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope_rotate_f32(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate rows ``x[i]`` (float32 ``[n, d]``) to ``positions[i]``; rotate-half pairing."""
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    C = d // 2
    inv_freq = theta ** (-2.0 * np.arange(C, dtype=np.float64) / d)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang).astype(np.float32)
    sin = np.sin(ang).astype(np.float32)
    return _rotate_with(x, cos, sin)


def _rotate_with(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    C = x.shape[-1] // 2
    x1 = x[:, :C]
    x2 = x[:, C:]
    out = np.empty_like(x)
    out[:, :C] = x1 * cos - x2 * sin
    out[:, C:] = x2 * cos + x1 * sin
    return out


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


# --------------------------------------------------------------------------------------
# presets: the five decode workloads, named by what they are
# --------------------------------------------------------------------------------------

PRESETS = {
    # batch 1, 1 layer, 4 q heads = 4 KV heads, d 64, L 512; KV heads 0-1 TIP+FAC, 2-3 sink 4 + window 60
    "tiny_mixed_d64_L512": WorkloadSpec(
        name="tiny_mixed_d64_L512", batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, theta=1e4,
        lengths=(512,), n_dom=4, n_fac=64,
        roles=(ROLE_SPARSE, ROLE_SPARSE, ROLE_STREAM, ROLE_STREAM), sink=4, window=60, seed=101),
    # Llama-3-8B-shaped layer: batch 4, 32/8 heads, d 128, L 32768, 1% planted keys, 16 of 64 chunks, N_fac 2048
    "llama8b_gqa4_L32k": WorkloadSpec(
        name="llama8b_gqa4_L32k", batch=4, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
        lengths=(32768,) * 4, n_dom=16, n_fac=2048, roles=(ROLE_SPARSE,) * 8,
        planted_frac=0.01, planted_gain=4.0, seed=202),
    # head-role split: batch 1, 32/8 heads, L 131072; 2 of 8 KV groups dense, 6 sink 128 + window 4096
    "aoh_roles_L128k": WorkloadSpec(
        name="aoh_roles_L128k", batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
        lengths=(131072,), n_retrieval=2, sink=128, window=4096, seed=303),
    # shared-index cross-decoder stack: batch 2, shared cache L 131072, 8 KV heads, 8 layers x 32 q heads, k 2048
    "clsa_shared_L128k": WorkloadSpec(
        name="clsa_shared_L128k", batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
        lengths=(131072,) * 2, n_layers=8, topk_shared=2048, seed=404),
    # batched serving: batch 64, L_b ~ U[4096, 65536], 28/4 heads, theta 1e6, N_fac = ceil(L_b / 8)
    "fasa_serving_ragged_b64": WorkloadSpec(
        name="fasa_serving_ragged_b64", batch=64, n_q_heads=28, n_kv_heads=4, head_dim=128, theta=1e6,
        len_range=(4096, 65536), n_dom=16, n_fac_div=8, roles=(ROLE_SPARSE,) * 4,
        planted_frac=0.01, planted_gain=4.0, seed=505),
}


def preset(name: str, **overrides) -> WorkloadSpec:
    spec = PRESETS[name]
    return replace(spec, **overrides) if overrides else spec


# --------------------------------------------------------------------------------------
# generation
# --------------------------------------------------------------------------------------

def _draw_lengths(spec: WorkloadSpec) -> np.ndarray:
    if spec.lengths is not None:
        assert len(spec.lengths) == spec.batch
        return np.asarray(spec.lengths, dtype=np.int64)
    lo, hi = spec.len_range
    return _rng(spec.seed, _TAG_LEN).integers(lo, hi, size=spec.batch, endpoint=True).astype(np.int64)


def _draw_idom(spec: WorkloadSpec) -> Optional[np.ndarray]:
    if spec.n_dom <= 0:
        return None
    C = spec.head_dim // 2
    out = np.empty((spec.n_kv_heads, spec.n_dom), dtype=np.int32)
    for g in range(spec.n_kv_heads):
        out[g] = np.sort(_rng(spec.seed, _TAG_IDOM, g).choice(C, spec.n_dom, replace=False))
    return out


def _draw_roles(spec: WorkloadSpec) -> np.ndarray:
    if spec.roles:
        assert len(spec.roles) == spec.n_kv_heads
        return np.asarray(spec.roles, dtype=np.uint8)
    if spec.n_retrieval >= 0:
        perm = _rng(spec.seed, _TAG_ROLE).permutation(spec.n_kv_heads)
        roles = np.full(spec.n_kv_heads, ROLE_STREAM, dtype=np.uint8)
        roles[perm[: spec.n_retrieval]] = ROLE_DENSE
        return roles
    return np.full(spec.n_kv_heads, ROLE_SPARSE, dtype=np.uint8)


def _n_fac(spec: WorkloadSpec, lengths: np.ndarray) -> np.ndarray:
    if spec.n_fac_div > 0:
        return np.array([-(-int(L) // spec.n_fac_div) for L in lengths], dtype=np.int32)
    if spec.topk_shared > 0:
        return np.full(spec.batch, spec.topk_shared, dtype=np.int32)
    return np.full(spec.batch, spec.n_fac, dtype=np.int32)


def planted_positions(spec: WorkloadSpec, b: int, g: int, L: int, idom_g: Optional[np.ndarray]):
    """Token positions and chunk ids boosted for (b, g): list of (t, chunk array)."""
    if spec.planted_frac <= 0 or idom_g is None or L == 0:
        return []
    rng = _rng(spec.seed, _TAG_PLANT, b, g)
    n_pl = int(math.ceil(spec.planted_frac * L))
    toks = np.sort(rng.choice(L, n_pl, replace=False))
    n_ch = int(math.ceil(len(idom_g) / 4))
    return [(int(t), np.sort(rng.choice(idom_g, n_ch, replace=False))) for t in toks]


def _key_block_raw(spec: WorkloadSpec, b: int, g: int, L: int, idom_g) -> Tuple[np.ndarray, list]:
    x = _rng(spec.seed, _TAG_K, b, g).standard_normal((L, spec.head_dim), dtype=np.float32)
    plants = planted_positions(spec, b, g, L, idom_g)
    C = spec.head_dim // 2
    for t, chunks in plants:
        x[t, chunks] *= np.float32(spec.planted_gain)
        x[t, chunks + C] *= np.float32(spec.planted_gain)
    return x, plants


def _value_block(spec: WorkloadSpec, b: int, g: int, L: int) -> np.ndarray:
    return _rng(spec.seed, _TAG_V, b, g).standard_normal((L, spec.head_dim), dtype=np.float32)


def query_raw(spec: WorkloadSpec, b: int, h: int, layer: int = -1, indexer: bool = False) -> np.ndarray:
    """Pre-rotation query vector (float32 [d]) of head h of sequence b."""
    if layer >= 0:
        rng = _rng(spec.seed, _TAG_QL, layer, b, h)
    elif indexer:
        rng = _rng(spec.seed, _TAG_QI, b, h)
    else:
        rng = _rng(spec.seed, _TAG_Q, b, h)
    return rng.standard_normal(spec.head_dim, dtype=np.float32)


def key_block_raw(spec: WorkloadSpec, b: int, g: int) -> np.ndarray:
    """Pre-rotation float32 keys [L_b, d] of (b, g), planted boosts included (for checks)."""
    lengths = _draw_lengths(spec)
    idom = _draw_idom(spec)
    x, _ = _key_block_raw(spec, b, g, int(lengths[b]), None if idom is None else idom[g])
    return x


def _n_threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def make_workload(spec: WorkloadSpec, threads: Optional[int] = None) -> Workload:
    """Generate every tensor of ``spec`` on the CPU (bf16 torch tensors, contiguous)."""
    B, Hq, Hkv, d = spec.batch, spec.n_q_heads, spec.n_kv_heads, spec.head_dim
    assert Hq % Hkv == 0 and d % 2 == 0
    lengths = _draw_lengths(spec)
    offsets = np.zeros(B + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(lengths)
    T = int(offsets[-1])
    assert T < 2**31
    idom = _draw_idom(spec)
    roles = _draw_roles(spec)
    Lmax = int(lengths.max()) if B else 0
    cos, sin = _angles(Lmax, d, spec.theta)

    k = torch.empty((T, Hkv, d), dtype=torch.bfloat16)
    v = torch.empty((T, Hkv, d), dtype=torch.bfloat16)
    planted = {}

    def fill(task):
        kind, b, g = task
        L = int(lengths[b])
        o = int(offsets[b])
        if L == 0:
            return
        if kind == 0:
            x, plants = _key_block_raw(spec, b, g, L, None if idom is None else idom[g])
            x = _rotate_with(x, cos[:L], sin[:L])
            k[o:o + L, g, :] = _to_bf16(x)
            planted[(b, g)] = np.array([t for t, _ in plants], dtype=np.int64)
        else:
            v[o:o + L, g, :] = _to_bf16(_value_block(spec, b, g, L))

    tasks = [(kind, b, g) for b in range(B) for g in range(Hkv) for kind in (0, 1)]
    nthr = threads or _n_threads()
    if nthr > 1 and len(tasks) > 1:
        with ThreadPoolExecutor(nthr) as ex:
            list(ex.map(fill, tasks))
    else:
        for t in tasks:
            fill(t)

    def q_tensor(layer: int = -1, indexer: bool = False) -> torch.Tensor:
        qa = np.empty((B, Hq, d), dtype=np.float32)
        for b in range(B):
            L = int(lengths[b])
            for h in range(Hq):
                qa[b, h] = rope_rotate_f32(query_raw(spec, b, h, layer, indexer)[None, :],
                                           np.array([L]), spec.theta)[0]
        return _to_bf16(qa)

    if spec.n_layers > 0:
        q = q_tensor(indexer=True)
        q_layers = torch.stack([q_tensor(layer=l) for l in range(spec.n_layers)])
    else:
        q = q_tensor()
        q_layers = None

    return Workload(
        spec=spec,
        lengths=lengths,
        offsets=torch.from_numpy(offsets.astype(np.int32)),
        k=k,
        v=v,
        q=q,
        q_layers=q_layers,
        idom=None if idom is None else torch.from_numpy(idom),
        roles=torch.from_numpy(roles),
        n_fac_per_seq=torch.from_numpy(_n_fac(spec, lengths)),
        scale=1.0 / math.sqrt(d),
        planted=planted,
    )


# --------------------------------------------------------------------------------------
# decoded tokens (appended one step at a time): raw rows, before any rotation
# --------------------------------------------------------------------------------------

_TAG_STEP = 10


def token_draws(seed: int, step: int, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int):
    """The new token of every sequence at decode step `step`: bf16 N(0,1) rows of its query
    [B, Hq, d], key [B, Hkv, d] and value [B, Hkv, d], as a model's projections would give
    them (before RoPE)."""
    r = _rng(seed, _TAG_STEP, step)
    q = r.standard_normal((batch, n_q_heads, head_dim), dtype=np.float32)
    k = r.standard_normal((batch, n_kv_heads, head_dim), dtype=np.float32)
    v = r.standard_normal((batch, n_kv_heads, head_dim), dtype=np.float32)
    return _to_bf16(q), _to_bf16(k), _to_bf16(v)


# --------------------------------------------------------------------------------------
# frozen projection weights for the head classifier (no trained checkpoint is used)
# --------------------------------------------------------------------------------------

_TAG_WQ, _TAG_WK, _TAG_BASIS, _TAG_RANKS = 11, 12, 13, 14


@dataclass(frozen=True)
class HeadWeightSpec:
    """Shape and recipe of synthetic q / k projection weights.

    Every KV group g gets a rank r_g (drawn from `ranks` by a seeded permutation; 0 means
    none): its key block and each of its q heads' blocks are `strength` times a rank-r_g
    product P R_g (P per head, R_g shared by the group, both N(0, 1)) plus unit N(0, 1)
    noise, all scaled by 1/sqrt(d_model) and rounded to bf16.  A small r_g concentrates
    the group's query-key spectrum; r_g = 0 leaves it as diffuse as noise.
    """

    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    d_model: int
    ranks: Tuple[int, ...]
    strength: float = 3.0
    n_retrieval: int = 0
    seed: int = 1


HEAD_WEIGHT_PRESETS = {
    # Llama-3-8B-shaped attention projections: 32 q / 8 KV heads of 128, d_model 4096; half the
    # KV groups retrieval heads (the pages' 50 % sparsity)
    "llama8b_heads": HeadWeightSpec(name="llama8b_heads", n_q_heads=32, n_kv_heads=8, head_dim=128, d_model=4096,
                                    ranks=(2, 4, 8, 16, 0, 0, 0, 0), n_retrieval=4, seed=606),
    # a small model: 8 q / 4 KV heads of 64, d_model 512
    "small_heads_d64": HeadWeightSpec(name="small_heads_d64", n_q_heads=8, n_kv_heads=4, head_dim=64, d_model=512,
                                      ranks=(3, 0, 12, 0), n_retrieval=2, seed=607),
}


def head_weights(spec: HeadWeightSpec):
    """(W_Q bf16 [Hq*d, d_model], W_K bf16 [Hkv*d, d_model], group ranks int64 [Hkv])."""
    Hq, Hkv, d, dm = spec.n_q_heads, spec.n_kv_heads, spec.head_dim, spec.d_model
    G = Hq // Hkv
    ranks = np.asarray(spec.ranks, dtype=np.int64)[_rng(spec.seed, _TAG_RANKS).permutation(Hkv)]
    scale = np.float32(1.0 / math.sqrt(dm))

    def block(tag, idx, g):
        r = _rng(spec.seed, tag, idx)
        w = r.standard_normal((d, dm), dtype=np.float32)
        if ranks[g] > 0:
            basis = _rng(spec.seed, _TAG_BASIS, g).standard_normal((int(ranks[g]), dm), dtype=np.float32)
            w += np.float32(spec.strength) * (r.standard_normal((d, int(ranks[g])), dtype=np.float32) @ basis)
        return w * scale

    wq = np.concatenate([block(_TAG_WQ, h, h // G) for h in range(Hq)])
    wk = np.concatenate([block(_TAG_WK, g, g) for g in range(Hkv)])
    return _to_bf16(wq), _to_bf16(wk), ranks
