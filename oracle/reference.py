"""Float64 CPU oracle of one token-sparse decode step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
executes this file: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs do.  It shares no code with the CUDA
path (no kernels, headers, tables or helpers); both sides only read the same
seeded bf16 inputs, which this module upcasts exactly to float64.

Sources (web-page summaries of the methods; section names as printed):

* FASA: Frequency-aware Sparse Attention -- §2.A (frequency chunks: RoPE splits
  a d-dim vector into d/2 orthogonal 2-D subspaces), §2.B.1 (Token Importance
  Predictor: a token's importance is the sum of the q.k contributions of the
  head's dominant chunks I_dom only; the N_fac best tokens are kept), §2.B.2
  (Focused Attention Computation: full-dimension attention over only those
  tokens, keeping their original absolute positions), §2.C (FASA-C keeps the
  whole cache on the GPU and reads only part of K).
* Resumen Técnico: Autonomía de Cabezales (AoH) -- Metodología §4 (retrieval
  heads keep the full global cache; streaming heads keep a fixed sink and a
  recent window; GQA scores are aggregated per group).
* El enrutamiento compartido entre capas ... (CLSA: You Only Index Once) --
  "Cómo funciona CLSA" (an indexer layer scores the cache once, takes the
  top-k once and hands the same index to every cross-decoder layer sharing
  that cache).
* Resumen Técnico: Por qué existen los patrones de atención (TAPPA) --
  "Mecanismos de Patrones Predictibles" (RoPE's relative-position property:
  shifting q and k together leaves their interaction unchanged).

Readings where the pages are silent (each is listed in the design notes):

* rotate-half RoPE layout: chunk c is the pair of dims (c, c + d/2), rotated by
  angle p * theta^(-2c/d);
* the importance score is computed on the rotated q and k, without the
  1/sqrt(d) scale, and summed over the q heads of a GQA group;
* ties in the top-N_fac go to the lower token position; selections are
  returned in ascending position order; N_fac >= L selects every token;
* the selection is the TIP top-N_fac only (no sink or window tokens added);
* a streaming head attends to positions [0, min(S, L)) U [max(0, L - W), L);
* q head h belongs to KV group h // G (contiguous GQA groups);
* the shared index is one top-k per (sequence, KV head) on full-dimension
  scores summed over the group, reused by every head of the group in every
  layer.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM = 0, 1, 2


# --------------------------------------------------------------------------------------
# RoPE frequency chunks (FASA §2.A)
# --------------------------------------------------------------------------------------

def rope(x: np.ndarray, positions: Sequence[float], theta: float) -> np.ndarray:
    """Rotate each row x[i] (float64 [n, d]) to absolute position positions[i].

    Chunk c = dims (c, c + d/2) is turned by angle positions[i] * theta^(-2c/d).
    """
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    C = d // 2
    out = np.empty_like(x)
    for c in range(C):
        w = theta ** (-2.0 * c / d)
        for i in range(n):
            a = float(positions[i]) * w
            ca, sa = math.cos(a), math.sin(a)
            u, v = x[i, c], x[i, c + C]
            out[i, c] = ca * u - sa * v
            out[i, c + C] = sa * u + ca * v
    return out


def dominant_dims(idom: Sequence[int], head_dim: int) -> List[int]:
    """The dims that the chunks in I_dom span: c and c + d/2 for every c."""
    C = head_dim // 2
    return [int(c) for c in idom] + [int(c) + C for c in idom]


# --------------------------------------------------------------------------------------
# Token Importance Predictor (FASA §2.B.1) with GQA group aggregation (AoH §4)
# --------------------------------------------------------------------------------------

def tip_scores(q_group: np.ndarray, keys: np.ndarray, idom: Sequence[int]) -> np.ndarray:
    """Importance of every cached token for one KV group.

    s[t] = sum over q heads h of the group, over chunks c in I_dom, of
           q_h[c] k_t[c] + q_h[c + C] k_t[c + C].
    q_group: [G, d]; keys: [L, d]; returns float64 [L].
    """
    q_group = np.asarray(q_group, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    d = keys.shape[1]
    C = d // 2
    s = np.zeros(keys.shape[0], dtype=np.float64)
    for h in range(q_group.shape[0]):
        for c in idom:
            c = int(c)
            s += q_group[h, c] * keys[:, c] + q_group[h, c + C] * keys[:, c + C]
    return s


# --------------------------------------------------------------------------------------
# top-N_fac selection (FASA §2.B.1; CLSA's single top-k)
# --------------------------------------------------------------------------------------

def select_top(scores: np.ndarray, n: int) -> np.ndarray:
    """Positions of the n highest scores, lower position first among equals; ascending output."""
    scores = np.asarray(scores)
    L = scores.shape[0]
    n = min(int(n), L)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    pos = np.arange(L)
    order = np.lexsort((pos, -scores.astype(np.float64)))  # primary: score desc; secondary: position asc
    return np.sort(order[:n]).astype(np.int64)


def tie_band(ref_scores: np.ndarray, n: int, rel: float = 1e-4, floor: float = 0.0) -> float:
    """Half-width beta of the score band around the n-th largest score s_n.

    beta = max(rel * |s_n|, floor).  The relative part is the band the selection may
    disagree within; `floor` is an absolute width a caller derives from the rounding
    bound of the scores it compares (an fp32 score cannot be closer than that to the
    exact one, so near s_n = 0 the relative band alone would demand the impossible).
    """
    s = np.asarray(ref_scores, dtype=np.float64)
    n = min(int(n), s.shape[0])
    if n <= 0:
        return float(floor)
    s_n = np.sort(s)[::-1][n - 1]
    return max(rel * abs(float(s_n)), float(floor))


def tie_band_check(gpu_sel: np.ndarray, ref_scores: np.ndarray, n: int, rel: float = 1e-4,
                   floor: float = 0.0) -> Tuple[bool, str]:
    """Is ``gpu_sel`` a valid top-n of ``ref_scores`` up to the score band around the n-th score?

    With s_n the n-th largest oracle score and beta = tie_band(ref_scores, n, rel, floor):
    every token with s > s_n + beta must be selected, none with s < s_n - beta,
    and exactly n tokens must be selected (each at most once).
    """
    s = np.asarray(ref_scores, dtype=np.float64)
    L = s.shape[0]
    n = min(int(n), L)
    sel = np.asarray(gpu_sel, dtype=np.int64)
    if sel.shape[0] != n:
        return False, f"selected {sel.shape[0]} tokens, expected {n}"
    if n == 0:
        return True, ""
    if np.any(sel < 0) or np.any(sel >= L):
        return False, "position out of range"
    if np.unique(sel).shape[0] != n:
        return False, "duplicate positions"
    if n == L:
        return True, ""
    s_n = np.sort(s)[::-1][n - 1]
    beta = tie_band(s, n, rel, floor)
    chosen = np.zeros(L, dtype=bool)
    chosen[sel] = True
    must = s > s_n + beta
    never = s < s_n - beta
    if np.any(must & ~chosen):
        return False, f"{int(np.sum(must & ~chosen))} tokens above the band missing"
    if np.any(never & chosen):
        return False, f"{int(np.sum(never & chosen))} tokens below the band selected"
    return True, ""


# --------------------------------------------------------------------------------------
# attention (FASA §2.B.2 focused attention; AoH §4 retrieval / streaming heads)
# --------------------------------------------------------------------------------------

def attend(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * keys @ q) @ values, in float64; empty key set -> zeros."""
    keys = np.asarray(keys, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1], dtype=np.float64)
    z = scale * (keys @ np.asarray(q, dtype=np.float64))
    p = np.exp(z - np.max(z))
    p /= np.sum(p)
    return p @ values


def focused_attention(q_group: np.ndarray, keys: np.ndarray, values: np.ndarray,
                      sel: np.ndarray, scale: float) -> np.ndarray:
    """Full-dimension attention of every q head of a group over the selected positions.

    The selected keys are used exactly as cached (rotated at their original
    positions); nothing is re-rotated.  Returns [G, d].
    """
    ks = np.asarray(keys, dtype=np.float64)[sel]
    vs = np.asarray(values, dtype=np.float64)[sel]
    return np.stack([attend(q_group[h], ks, vs, scale) for h in range(q_group.shape[0])])


def stream_positions(L: int, sink: int, window: int) -> np.ndarray:
    """Sink tokens [0, min(S, L)) together with the recent window [max(0, L - W), L)."""
    keep = set(range(0, min(sink, L))) | set(range(max(0, L - window), L))
    return np.array(sorted(keep), dtype=np.int64)


def dense_positions(L: int) -> np.ndarray:
    return np.arange(L, dtype=np.int64)


# --------------------------------------------------------------------------------------
# cache maintenance: appending the decoded token (AoH §4: retrieval heads keep the whole
# cache, streaming heads keep only a fixed sink and a recent window; FASA §2.C: the
# dominant part of K is kept apart)
# --------------------------------------------------------------------------------------

def ring_slot(p: int, sink: int, window: int) -> int:
    """Slot of position p in a streaming head's cache of sink + window slots.

    Positions below the sink keep their own slot; later positions take the window
    slots in turn, each overwriting the position `window` places before it.
    Returns -1 when the head keeps no window (window = 0) and p >= sink.
    """
    if p < sink:
        return p
    if window == 0:
        return -1
    return sink + (p - sink) % window


def ring_contents(L: int, sink: int, window: int) -> np.ndarray:
    """Position held by every slot after positions 0 .. L-1 were written in order (-1: empty)."""
    slots = np.full(sink + window, -1, dtype=np.int64)
    for p in range(L):
        s = ring_slot(p, sink, window)
        if s >= 0:
            slots[s] = p
    return slots


def to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to bf16 storage: to float32 (nearest), then to 8 significant
    bits, nearest with ties to even.  Returns the uint16 bit patterns (finite inputs)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact float64 value of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def append_token_rows(q_raw: np.ndarray, k_raw: np.ndarray, v_raw: np.ndarray, position: int,
                      theta: float) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Rows a decoded token adds: its query and key rotated to `position` (FASA §2.A
    chunks), its value as given; all rounded to bf16 (bit patterns).

    q_raw: [Hq, d]; k_raw, v_raw: [Hkv, d] (pre-rotation values).  The key is stored at
    `position` = the number of tokens the sequence held before; the query sits at the
    same position.
    """
    q = rope(np.asarray(q_raw, dtype=np.float64), [position] * len(q_raw), theta)
    k = rope(np.asarray(k_raw, dtype=np.float64), [position] * len(k_raw), theta)
    return to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(np.asarray(v_raw, dtype=np.float64))


def rest_dims(idom: Sequence[int], head_dim: int) -> List[int]:
    """The dims outside the dominant chunks, ascending: what FASA-M (§2.C) moves to host memory
    together with V, while the dominant components of K stay on the GPU."""
    dom = set(dominant_dims(idom, head_dim))
    return [i for i in range(head_dim) if i not in dom]


def pack_dominant_row(k_row: np.ndarray, idom: Sequence[int], cols: int) -> np.ndarray:
    """The dominant columns of one key row: dims I_dom, then dims I_dom + d/2, zero-padded to cols."""
    k_row = np.asarray(k_row)
    dims = dominant_dims(idom, k_row.shape[0])
    out = np.zeros(cols, dtype=k_row.dtype)
    out[:len(dims)] = k_row[dims]
    return out


# --------------------------------------------------------------------------------------
# AoH head classifier (AoH summary, Metodología §1-§4): the effective rank of every head's
# frozen query-key kernel, computed from its d_head x d_head proxy, aggregated per GQA
# group; the lowest become retrieval heads
# --------------------------------------------------------------------------------------

def head_rows(W: np.ndarray, h: int, head_dim: int) -> np.ndarray:
    """Head h's block of a projection weight [H * d_head, d_model]: rows h*d_head .. (h+1)*d_head."""
    return np.asarray(W, dtype=np.float64)[h * head_dim:(h + 1) * head_dim]


def qk_kernel(wq: np.ndarray, wk: np.ndarray) -> np.ndarray:
    """M_h = W_K^T W_Q (d_model x d_model) for head blocks wq, wk [d_head, d_model] (§1)."""
    return np.asarray(wk, dtype=np.float64).T @ np.asarray(wq, dtype=np.float64)


def proxy_matrix(wq: np.ndarray, wk: np.ndarray) -> np.ndarray:
    """C_h = (W_Q W_Q^T)(W_K W_K^T), d_head x d_head (§3)."""
    wq = np.asarray(wq, dtype=np.float64)
    wk = np.asarray(wk, dtype=np.float64)
    return (wq @ wq.T) @ (wk @ wk.T)


def proxy_singular_values(wq: np.ndarray, wk: np.ndarray) -> np.ndarray:
    """Singular values of M_h from the proxy (§3, Sylvester): sigma_k = sqrt(eig_k(C_h)).

    C_h is a product of two positive semi-definite matrices, so its eigenvalues are real
    and non-negative; rounding leaves tiny imaginary parts and negatives, dropped here.
    Returned in descending order.
    """
    lam = np.linalg.eigvals(proxy_matrix(wq, wk)).real
    return np.sort(np.sqrt(np.maximum(lam, 0.0)))[::-1]


def effective_rank(sigma: np.ndarray, rel_zero: float = 1e-12) -> float:
    """exp of the Shannon entropy of the normalised non-zero singular values (§2).

    sigma_hat_k = sigma_k / sum sigma over the r_h non-zero values (those above
    rel_zero * max sigma), ER = exp(-sum sigma_hat_k log sigma_hat_k).
    """
    s = np.asarray(sigma, dtype=np.float64)
    if s.size == 0 or s.max() <= 0:
        return 0.0
    s = s[s > rel_zero * s.max()]
    p = s / s.sum()
    return float(np.exp(-np.sum(p * np.log(p))))


def head_effective_ranks(W_Q: np.ndarray, W_K: np.ndarray, n_q_heads: int, n_kv_heads: int,
                         head_dim: int) -> np.ndarray:
    """ER of every q head h, whose key block is KV head h // G (GQA): float64 [n_q_heads]."""
    G = n_q_heads // n_kv_heads
    return np.array([effective_rank(proxy_singular_values(head_rows(W_Q, h, head_dim),
                                                          head_rows(W_K, h // G, head_dim)))
                     for h in range(n_q_heads)])


def group_effective_ranks(er_heads: np.ndarray, n_kv_heads: int) -> np.ndarray:
    """GQA aggregation by the mean (§4): the mean ER of each group's q heads, float64 [n_kv_heads]."""
    er = np.asarray(er_heads, dtype=np.float64)
    G = er.shape[0] // n_kv_heads
    return np.array([er[g * G:(g + 1) * G].mean() for g in range(n_kv_heads)])


def classify_heads(er_groups: np.ndarray, n_retrieval: int) -> np.ndarray:
    """Roles per KV head (§4): the n_retrieval lowest-ER groups are retrieval heads (DENSE,
    the whole cache), the rest streaming heads (STREAM); equal ER: the lower index first."""
    er = np.asarray(er_groups, dtype=np.float64)
    order = np.lexsort((np.arange(er.shape[0]), er))
    roles = np.full(er.shape[0], ROLE_STREAM, dtype=np.uint8)
    roles[order[:max(0, int(n_retrieval))]] = ROLE_DENSE
    return roles


# --------------------------------------------------------------------------------------
# one decode step
# --------------------------------------------------------------------------------------

def decode_row(q_group: np.ndarray, keys: np.ndarray, values: np.ndarray, role: int, scale: float,
               idom: Optional[Sequence[int]] = None, n_fac: int = 0,
               sink: int = 0, window: int = 0) -> Dict[str, np.ndarray]:
    """Decode-step output of one (sequence, KV group) by head role.

    SPARSE: TIP scores -> top-N_fac -> focused attention; DENSE: attention over
    the whole cache; STREAM: attention over the sink + recent window.
    Returns {"out": [G, d], "sel": positions used, "scores": TIP scores or None}.
    """
    L = keys.shape[0]
    if role == ROLE_SPARSE:
        s = tip_scores(q_group, keys, idom)
        sel = select_top(s, n_fac)
        return {"out": focused_attention(q_group, keys, values, sel, scale), "sel": sel, "scores": s}
    if role == ROLE_DENSE:
        sel = dense_positions(L)
    elif role == ROLE_STREAM:
        sel = stream_positions(L, sink, window)
    else:
        raise ValueError(f"unknown role {role}")
    return {"out": focused_attention(q_group, keys, values, sel, scale), "sel": sel, "scores": None}


def decode_step(q: np.ndarray, k: np.ndarray, v: np.ndarray, offsets: Sequence[int], roles: Sequence[int],
                scale: float, idom: Optional[np.ndarray] = None, n_fac_per_seq: Optional[Sequence[int]] = None,
                sink: int = 0, window: int = 0,
                rows: Optional[Sequence[Tuple[int, int]]] = None) -> Dict[Tuple[int, int], Dict[str, np.ndarray]]:
    """Every (b, g) row of one decode step (or only ``rows``).

    q: [B, Hq, d]; k, v: [T_total, Hkv, d]; offsets: [B + 1].
    """
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if rows is None:
        rows = [(b, g) for b in range(B) for g in range(Hkv)]
    res = {}
    for b, g in rows:
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        res[(b, g)] = decode_row(
            np.asarray(q[b, g * G:(g + 1) * G], dtype=np.float64),
            np.asarray(k[o0:o1, g], dtype=np.float64), np.asarray(v[o0:o1, g], dtype=np.float64),
            int(roles[g]), scale,
            None if idom is None else idom[g], 0 if n_fac_per_seq is None else int(n_fac_per_seq[b]),
            sink, window)
    return res


def shared_index_step(q_index: np.ndarray, q_layers: np.ndarray, k: np.ndarray, v: np.ndarray,
                      offsets: Sequence[int], topk: int, scale: float,
                      rows: Optional[Sequence[Tuple[int, int]]] = None) -> Dict[Tuple[int, int], Dict[str, np.ndarray]]:
    """Shared-index cross-decoder stack: index once, reuse in every layer.

    The indexer's full-dimension scores (every chunk, summed over the group's
    q heads) give one top-k per (sequence, KV group); each layer l then runs
    focused attention of its own q over those positions of the shared cache.
    q_index: [B, Hq, d]; q_layers: [n_layers, B, Hq, d].
    Returns {(b, g): {"sel", "scores", "out": [n_layers, G, d]}}.
    """
    n_layers, B, Hq, d = q_layers.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    all_chunks = list(range(d // 2))
    if rows is None:
        rows = [(b, g) for b in range(B) for g in range(Hkv)]
    res = {}
    for b, g in rows:
        o0, o1 = int(offsets[b]), int(offsets[b + 1])
        keys = np.asarray(k[o0:o1, g], dtype=np.float64)
        vals = np.asarray(v[o0:o1, g], dtype=np.float64)
        s = tip_scores(np.asarray(q_index[b, g * G:(g + 1) * G], dtype=np.float64), keys, all_chunks)
        sel = select_top(s, topk)
        out = np.stack([focused_attention(np.asarray(q_layers[l, b, g * G:(g + 1) * G], dtype=np.float64),
                                          keys, vals, sel, scale) for l in range(n_layers)])
        res[(b, g)] = {"sel": sel, "scores": s, "out": out}
    return res
