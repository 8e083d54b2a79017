"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle (on the CPU, through monkeypatch: the
oracle package and its module both see the mutant) and runs every pin of
test_oracle_pins.py; at least one pin must fail.  The mutants are the mistakes a
restatement of the method could plausibly make: a RoPE rotation of the wrong
sense, the wrong pairing of dims or a wrong frequency; a TIP that drops the
c + d/2 term or scores one head of the group; a select that breaks ties toward
the higher position or returns positions in score order; attention without the
scale or with keys where values belong; a streaming window one token short; a ring
slot one place off, bf16 storage by truncation, a token appended one position
late, dominant columns packed in the wrong half order; a head classifier that takes
the proxy's eigenvalues for singular values, a base-2 entropy, the group maximum for
the mean, or the highest ranks for retrieval heads.
"""

import inspect
import json
import math
import os

import numpy as np
import pytest

import oracle
import oracle.reference as ref
import test_oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def rope_wrong_sense(x, positions, theta):
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
            out[i, c] = ca * u + sa * v
            out[i, c + C] = -sa * u + ca * v
    return out


def rope_interleaved(x, positions, theta):
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    out = np.empty_like(x)
    for c in range(d // 2):
        w = theta ** (-2.0 * c / d)
        for i in range(n):
            a = float(positions[i]) * w
            ca, sa = math.cos(a), math.sin(a)
            u, v = x[i, 2 * c], x[i, 2 * c + 1]
            out[i, 2 * c] = ca * u - sa * v
            out[i, 2 * c + 1] = sa * u + ca * v
    return out


def rope_half_frequency(x, positions, theta):
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    C = d // 2
    out = np.empty_like(x)
    for c in range(C):
        w = theta ** (-1.0 * c / d)
        for i in range(n):
            a = float(positions[i]) * w
            ca, sa = math.cos(a), math.sin(a)
            u, v = x[i, c], x[i, c + C]
            out[i, c] = ca * u - sa * v
            out[i, c + C] = sa * u + ca * v
    return out


def tip_first_half_only(q_group, keys, idom):
    q_group = np.asarray(q_group, dtype=np.float64)
    keys = np.asarray(keys, dtype=np.float64)
    s = np.zeros(keys.shape[0])
    for h in range(q_group.shape[0]):
        for c in idom:
            s += q_group[h, int(c)] * keys[:, int(c)]
    return s


def tip_one_head(q_group, keys, idom):
    return ref.__wrapped_tip(np.asarray(q_group)[:1], keys, idom)


def select_ties_high(scores, n):
    scores = np.asarray(scores)
    L = scores.shape[0]
    n = min(int(n), L)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    order = np.lexsort((-np.arange(L), -scores.astype(np.float64)))
    return np.sort(order[:n]).astype(np.int64)


def select_score_order(scores, n):
    scores = np.asarray(scores)
    L = scores.shape[0]
    n = min(int(n), L)
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    return np.lexsort((np.arange(L), -scores.astype(np.float64)))[:n].astype(np.int64)


def attend_no_scale(q, keys, values, scale):
    return ref.__wrapped_attend(q, keys, values, 1.0)


def attend_keys_for_values(q, keys, values, scale):
    return ref.__wrapped_attend(q, keys, keys, scale)


def stream_window_short(L, sink, window):
    keep = set(range(0, min(sink, L))) | set(range(max(0, L - window + 1), L))
    return np.array(sorted(keep), dtype=np.int64)


def ring_slot_off_by_one(p, sink, window):
    if p < sink:
        return p
    if window == 0:
        return -1
    return sink + (p - sink + 1) % window


def bf16_truncate(x):
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def append_one_late(q_raw, k_raw, v_raw, position, theta):
    return ref.__wrapped_append(q_raw, k_raw, v_raw, position + 1, theta)


def pack_second_half_first(k_row, idom, cols):
    k_row = np.asarray(k_row)
    C = k_row.shape[0] // 2
    dims = [int(c) + C for c in idom] + [int(c) for c in idom]
    out = np.zeros(cols, dtype=k_row.dtype)
    out[:len(dims)] = k_row[dims]
    return out


def proxy_eigenvalues_not_roots(wq, wk):
    lam = np.linalg.eigvals(ref.proxy_matrix(wq, wk)).real
    return np.sort(np.maximum(lam, 0.0))[::-1]


def effective_rank_log2(sigma, rel_zero=1e-12):
    s = np.asarray(sigma, dtype=np.float64)
    if s.size == 0 or s.max() <= 0:
        return 0.0
    s = s[s > rel_zero * s.max()]
    p = s / s.sum()
    return float(np.exp(-np.sum(p * np.log2(p))))


def group_max(er_heads, n_kv_heads):
    er = np.asarray(er_heads, dtype=np.float64)
    G = er.shape[0] // n_kv_heads
    return np.array([er[g * G:(g + 1) * G].max() for g in range(n_kv_heads)])


def classify_highest(er_groups, n_retrieval):
    er = np.asarray(er_groups, dtype=np.float64)
    order = np.lexsort((np.arange(er.shape[0]), -er))
    roles = np.full(er.shape[0], ref.ROLE_STREAM, dtype=np.uint8)
    roles[order[:max(0, int(n_retrieval))]] = ref.ROLE_DENSE
    return roles


def rest_dims_drops_last(idom, head_dim):
    return ref.__wrapped_rest(idom, head_dim)[:-1]


MUTANTS = {
    "rope_wrong_sense": ("rope", rope_wrong_sense),
    "rope_interleaved_pairs": ("rope", rope_interleaved),
    "rope_half_frequency": ("rope", rope_half_frequency),
    "tip_drops_c_plus_half": ("tip_scores", tip_first_half_only),
    "tip_scores_one_head": ("tip_scores", tip_one_head),
    "select_ties_to_higher_position": ("select_top", select_ties_high),
    "select_in_score_order": ("select_top", select_score_order),
    "attend_without_scale": ("attend", attend_no_scale),
    "attend_keys_as_values": ("attend", attend_keys_for_values),
    "stream_window_one_short": ("stream_positions", stream_window_short),
    "ring_slot_off_by_one": ("ring_slot", ring_slot_off_by_one),
    "bf16_truncates": ("to_bf16_bits", bf16_truncate),
    "append_one_position_late": ("append_token_rows", append_one_late),
    "pack_second_half_first": ("pack_dominant_row", pack_second_half_first),
    "proxy_eigenvalues_as_singular_values": ("proxy_singular_values", proxy_eigenvalues_not_roots),
    "effective_rank_base_two": ("effective_rank", effective_rank_log2),
    "group_by_max": ("group_effective_ranks", group_max),
    "retrieval_is_highest_rank": ("classify_heads", classify_highest),
    "rest_dims_drops_one": ("rest_dims", rest_dims_drops_last),
}


def run_pins():
    """Names of the pins that fail (any exception) with the oracle as it is now."""
    with open(GOLDEN) as f:
        hand = json.load(f)
    failed = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        args = [hand if p == "hand" else None for p in inspect.signature(fn).parameters]
        try:
            fn(*args)
        except Exception:  # an assertion, or a shape error the mistake causes
            failed.append(name)
    return failed


def test_unmutated_oracle_passes_every_pin():
    assert run_pins() == []


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutant_is_caught(mutant, monkeypatch):
    attr, fn = MUTANTS[mutant]
    # helpers some mutants call: the original functions
    monkeypatch.setattr(ref, "__wrapped_tip", ref.tip_scores, raising=False)
    monkeypatch.setattr(ref, "__wrapped_attend", ref.attend, raising=False)
    monkeypatch.setattr(ref, "__wrapped_append", ref.append_token_rows, raising=False)
    monkeypatch.setattr(ref, "__wrapped_rest", ref.rest_dims, raising=False)
    monkeypatch.setattr(ref, attr, fn)
    monkeypatch.setattr(oracle, attr, fn)
    failed = run_pins()
    assert failed, f"no pin catches the mutant {mutant}"
