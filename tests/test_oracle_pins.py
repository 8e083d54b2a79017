"""Pins of the float64 oracle to facts other than itself.

Each test checks the oracle against a closed form, a hand-worked example, an
independent library routine on a special case, an invariant of the mathematics
or brute force on tiny inputs, so that a dropped term, a wrong sign, a wrong
pairing of RoPE dims or a transposed operand fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
from oracle.reference import ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


@pytest.fixture(scope="module")
def hand():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------------------- RoPE chunks

def test_rope_quarter_turn_closed_form():
    # d = 2: a single chunk with frequency theta^0 = 1; position pi/2 turns (1, 0) into (0, 1).
    out = oracle.rope(np.array([[1.0, 0.0]]), [math.pi / 2], 1e4)
    assert np.allclose(out, [[0.0, 1.0]], atol=1e-15)


def test_rope_pairs_dim_c_with_c_plus_half():
    # d = 4, theta = 100: chunk 1 (dims 1 and 3) has frequency 100^(-1/2) = 0.1;
    # position 5*pi is a quarter turn for it, so one-hot dim 1 lands on dim 3 and nowhere else.
    x = np.array([[0.0, 1.0, 0.0, 0.0]])
    out = oracle.rope(x, [5 * math.pi], 100.0)
    assert np.allclose(out, [[0.0, 0.0, 0.0, 1.0]], atol=1e-14)
    # chunk 0 (dims 0 and 2) has frequency 1: position pi flips its sign.
    out0 = oracle.rope(np.array([[1.0, 0.0, 0.0, 0.0]]), [math.pi], 100.0)
    assert np.allclose(out0, [[-1.0, 0.0, 0.0, 0.0]], atol=1e-14)


def test_rope_full_period_is_identity_and_norm_per_chunk():
    rng = np.random.default_rng(0)
    d, theta = 16, 1e4
    x = rng.standard_normal((1, d))
    C = d // 2
    for c in range(C):
        period = 2 * math.pi / theta ** (-2.0 * c / d)
        y = oracle.rope(x, [period], theta)
        # chunk c is back where it started
        assert np.allclose(y[0, [c, c + C]], x[0, [c, c + C]], rtol=1e-9, atol=1e-9)
    y = oracle.rope(x, [123.0], theta)
    for c in range(C):
        assert math.isclose(np.hypot(y[0, c], y[0, c + C]), np.hypot(x[0, c], x[0, c + C]), rel_tol=1e-13)


def test_rope_relative_position_invariance():
    # Shifting q and k by the same amount leaves q.k unchanged (RoPE's relative-position property).
    rng = np.random.default_rng(1)
    d, theta = 64, 1e4
    q = rng.standard_normal((1, d))
    ks = rng.standard_normal((5, d))
    m, ns = 512.0, [0.0, 3.0, 100.0, 400.0, 511.0]
    base = oracle.rope(ks, ns, theta) @ oracle.rope(q, [m], theta)[0]
    for delta in [1.0, 17.0, 1000.0, 65536.0]:
        moved = oracle.rope(ks, [n + delta for n in ns], theta) @ oracle.rope(q, [m + delta], theta)[0]
        assert np.allclose(moved, base, rtol=1e-9, atol=1e-9)
    # and it is not invariant to moving only one of them
    moved_k = oracle.rope(ks, [n + 7.0 for n in ns], theta) @ oracle.rope(q, [m], theta)[0]
    assert not np.allclose(moved_k, base, rtol=1e-3)


def test_generator_rotation_agrees_with_oracle_rope():
    # The input generator's float32 rotation and the oracle's float64 one are two separate
    # implementations of the same map.
    from workloads import rope_rotate_f32

    rng = np.random.default_rng(2)
    for d, theta in [(64, 1e4), (128, 5e5), (128, 1e6)]:
        x = rng.standard_normal((6, d)).astype(np.float32)
        pos = np.array([0, 1, 77, 4095, 32767, 131071])
        a = rope_rotate_f32(x, pos, theta).astype(np.float64)
        b = oracle.rope(x.astype(np.float64), pos, theta)
        assert np.allclose(a, b, rtol=0, atol=1e-5 * np.abs(x).max())


# ---------------------------------------------------------------------------- TIP scores

def test_tip_hand_example(hand):
    q = np.array(hand["q_group"], dtype=np.float64)
    k = np.array(hand["keys"], dtype=np.float64)
    assert np.array_equal(oracle.tip_scores(q, k, hand["idom"]), hand["tip_scores"])
    assert np.array_equal(oracle.tip_scores(q, k, [0, 1]), hand["full_scores"])


def test_tip_all_chunks_equals_full_dot():
    rng = np.random.default_rng(3)
    for G, d, L in [(1, 64, 50), (4, 128, 300), (7, 128, 33)]:
        q = rng.standard_normal((G, d))
        k = rng.standard_normal((L, d))
        s = oracle.tip_scores(q, k, range(d // 2))
        ref = np.dot(k, q.sum(axis=0))
        assert np.allclose(s, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_tip_is_linear_in_the_group():
    rng = np.random.default_rng(4)
    G, d, L = 4, 128, 200
    q = rng.standard_normal((G, d))
    k = rng.standard_normal((L, d))
    idom = np.sort(rng.choice(d // 2, 16, replace=False))
    per_head = sum(oracle.tip_scores(q[h:h + 1], k, idom) for h in range(G))
    assert np.allclose(oracle.tip_scores(q, k, idom), per_head, rtol=1e-12, atol=1e-12)


def test_tip_one_hot_query_reads_exactly_the_dominant_dims():
    rng = np.random.default_rng(5)
    d, L = 16, 9
    C = d // 2
    k = rng.standard_normal((L, d))
    idom = [1, 5]
    dims = set(oracle.dominant_dims(idom, d))
    assert dims == {1, 5, 1 + C, 5 + C}
    for i in range(d):
        q = np.zeros((1, d))
        q[0, i] = 1.0
        s = oracle.tip_scores(q, k, idom)
        if i in dims:
            assert np.array_equal(s, k[:, i])
        else:
            assert np.array_equal(s, np.zeros(L))


# ---------------------------------------------------------------------------- selection

def _brute_force_top(scores, n):
    """The unique n-subset whose every member beats every outsider (score desc, position asc)."""
    L = len(scores)
    better = lambda a, b: scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
    found = []
    for sub in itertools.combinations(range(L), n):
        inside = set(sub)
        if all(better(a, b) for a in inside for b in range(L) if b not in inside):
            found.append(sub)
    assert len(found) == 1
    return np.array(found[0])


def test_select_matches_brute_force_on_tiny_rows():
    rng = np.random.default_rng(6)
    for trial in range(60):
        L = int(rng.integers(1, 11))
        # small integer scores so that ties are frequent
        s = rng.integers(-3, 4, size=L).astype(np.float64)
        for n in range(0, L + 1):
            got = oracle.select_top(s, n)
            if n == 0:
                assert got.size == 0
                continue
            assert np.array_equal(got, _brute_force_top(s, n)), (s, n)


def test_select_hand_example(hand):
    s = np.array(hand["tip_scores"], dtype=np.float64)
    assert list(oracle.select_top(s, 2)) == hand["top2"]
    assert list(oracle.select_top(s, 3)) == hand["top3"]
    assert list(oracle.select_top(np.array(hand["full_scores"], float), 2)) == hand["full_top2"]


def test_select_special_cases():
    assert list(oracle.select_top(np.zeros(10), 4)) == [0, 1, 2, 3]          # all equal -> lowest positions
    assert list(oracle.select_top(np.array([1.0, 2.0, 2.0, 1.0]), 1)) == [1]  # duplicate maximum -> lower
    assert list(oracle.select_top(np.array([3.0, 1.0, 2.0]), 10)) == [0, 1, 2]  # N_fac >= L -> everything
    assert list(oracle.select_top(np.array([-0.0, 0.0, -1.0]), 1)) == [0]     # -0 and +0 are equal scores


def test_tie_band_check_accepts_and_rejects():
    s = np.array([10.0, 5.0, 5.0000001, 1.0, 0.0])
    assert oracle.tie_band_check(np.array([0, 2]), s, 2)[0]
    assert oracle.tie_band_check(np.array([0, 1]), s, 2)[0]       # swap inside the band
    assert not oracle.tie_band_check(np.array([0, 3]), s, 2)[0]   # token below the band
    assert not oracle.tie_band_check(np.array([1, 2]), s, 2)[0]   # token above the band missing
    assert not oracle.tie_band_check(np.array([0]), s, 2)[0]      # wrong count
    assert not oracle.tie_band_check(np.array([0, 0]), s, 2)[0]   # duplicate


def test_tie_band_is_relative_to_the_nth_score_with_a_floor():
    # n = 3, s_n = 5: beta = 1e-4 * 5 = 5e-4 (the far-off scores do not enter it)
    s = np.array([1000.0, 10.0, 5.0, 4.9996, -1000.0])
    assert oracle.tie_band(s, 3) == pytest.approx(5e-4)
    assert oracle.tie_band_check(np.array([0, 1, 2]), s, 3)[0]
    assert oracle.tie_band_check(np.array([0, 1, 3]), s, 3)[0]       # 4.9996 is inside the band
    s2 = np.array([1000.0, 10.0, 5.0, 4.9994, -1000.0])
    assert not oracle.tie_band_check(np.array([0, 1, 3]), s2, 3)[0]  # 4.9994 < 5 - 5e-4: below it
    # s_n = 0: the relative band is empty, only the caller's rounding floor remains
    z = np.array([3.0, 1e-9, 0.0, -1e-9, -2.0])
    assert oracle.tie_band(z, 3) == 0.0
    assert not oracle.tie_band_check(np.array([0, 1, 3]), z, 3)[0]
    assert oracle.tie_band_check(np.array([0, 1, 3]), z, 3, floor=1e-8)[0]
    assert oracle.tie_band(z, 3, floor=1e-8) == 1e-8


# ---------------------------------------------------------------------------- attention

def test_attend_hand_example(hand):
    a = hand["attention"]
    k = np.array(hand["keys"], dtype=np.float64)
    v = np.array(a["values"], dtype=np.float64)
    sel = np.array(a["selected"])
    out = oracle.focused_attention(np.array([a["q"]], float), k, v, sel, a["scale"])
    assert np.allclose(out[0], a["out"], rtol=1e-15, atol=1e-15)


def test_attend_two_tokens_is_logistic():
    rng = np.random.default_rng(7)
    for _ in range(20):
        q, k1, k2, v1, v2 = rng.standard_normal((5, 8))
        z1, z2 = 0.3 * k1 @ q, 0.3 * k2 @ q
        w1 = 1.0 / (1.0 + math.exp(-(z1 - z2)))
        ref = w1 * v1 + (1.0 - w1) * v2
        assert np.allclose(oracle.attend(q, np.stack([k1, k2]), np.stack([v1, v2]), 0.3), ref, rtol=1e-13, atol=1e-14)


def test_attend_weights_match_library_softmax_and_sum_to_one():
    rng = np.random.default_rng(8)
    L, d = 40, 16
    q, k = rng.standard_normal(d), rng.standard_normal((L, d))
    # values = identity rows -> the output is the weight vector itself
    p = oracle.attend(q, k, np.eye(L), 0.25)
    assert np.allclose(p, scipy.special.softmax(0.25 * k @ q), rtol=1e-12, atol=1e-15)
    assert math.isclose(oracle.attend(q, k, np.ones((L, 1)), 0.25)[0], 1.0, rel_tol=1e-14)


def test_attend_dominant_key():
    rng = np.random.default_rng(9)
    L, d = 30, 16
    q = rng.standard_normal(d)
    k = rng.standard_normal((L, d)) * 0.1
    v = rng.standard_normal((L, d))
    k[17] = q * (60.0 / (q @ q))            # logit margin ~ 60 over every other key
    assert np.allclose(oracle.attend(q, k, v, 1.0), v[17], rtol=0, atol=1e-12)


def test_focused_with_every_token_is_dense():
    rng = np.random.default_rng(10)
    G, d, L = 4, 32, 57
    q = rng.standard_normal((G, d))
    k, v = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    idom = [0, 3, 9]
    res = oracle.decode_row(q, k, v, ROLE_SPARSE, 0.2, idom=idom, n_fac=L + 5)
    dense = scipy.special.softmax(0.2 * q @ k.T, axis=1) @ v
    assert np.allclose(res["out"], dense, rtol=1e-12, atol=1e-13)
    assert np.array_equal(res["sel"], np.arange(L))


def test_focused_keeps_original_positions():
    # Re-rotating the selected keys at compacted positions 0..n-1 is a different (wrong) computation.
    rng = np.random.default_rng(11)
    d, L, theta = 32, 64, 1e4
    raw_k = rng.standard_normal((L, d))
    raw_q = rng.standard_normal((1, d))
    v = rng.standard_normal((L, d))
    k = oracle.rope(raw_k, range(L), theta)
    q = oracle.rope(raw_q, [L], theta)
    sel = np.array([2, 9, 30, 31, 50, 63])
    right = oracle.focused_attention(q, k, v, sel, 0.3)
    k_wrong = oracle.rope(raw_k[sel], range(len(sel)), theta)
    wrong = oracle.focused_attention(q, k_wrong, v[sel], np.arange(len(sel)), 0.3)
    assert not np.allclose(right, wrong, atol=1e-3)


# ---------------------------------------------------------------------------- head roles

def test_stream_positions_hand_example(hand):
    st = hand["stream"]
    assert list(oracle.stream_positions(st["L"], st["sink"], st["window"])) == st["positions"]
    assert list(oracle.stream_positions(10, 0, 0)) == []
    assert list(oracle.stream_positions(10, 4, 8)) == list(range(10))   # S + W >= L -> dense
    assert list(oracle.stream_positions(3, 128, 4096)) == [0, 1, 2]


def test_stream_head_is_masked_dense_attention():
    rng = np.random.default_rng(12)
    G, d, L, S, W = 2, 16, 90, 5, 20
    q = rng.standard_normal((G, d))
    k, v = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    res = oracle.decode_row(q, k, v, ROLE_STREAM, 0.25, sink=S, window=W)
    mask = np.full(L, -np.inf)
    mask[:S] = 0.0
    mask[L - W:] = 0.0
    ref = scipy.special.softmax(0.25 * q @ k.T + mask[None, :], axis=1) @ v
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-13)
    dense = oracle.decode_row(q, k, v, ROLE_DENSE, 0.25)
    wide = oracle.decode_row(q, k, v, ROLE_STREAM, 0.25, sink=50, window=40)
    assert np.allclose(dense["out"], wide["out"], rtol=1e-13, atol=1e-14)


def test_decode_step_gqa_groups_are_contiguous():
    # q head h reads KV group h // G: with G = 2, heads 2 and 3 use KV group 1.
    rng = np.random.default_rng(13)
    B, Hq, Hkv, d, L = 1, 4, 2, 16, 12
    q = rng.standard_normal((B, Hq, d))
    k, v = rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d))
    res = oracle.decode_step(q, k, v, [0, L], [ROLE_DENSE, ROLE_DENSE], 0.25)
    for h in range(Hq):
        ref = scipy.special.softmax(0.25 * k[:, h // 2] @ q[0, h]) @ v[:, h // 2]
        assert np.allclose(res[(0, h // 2)]["out"][h % 2], ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------- shared index

def test_shared_index_with_k_equal_L_is_dense_in_every_layer():
    rng = np.random.default_rng(14)
    n_layers, B, Hq, Hkv, d, L = 3, 2, 4, 2, 16, 20
    qi = rng.standard_normal((B, Hq, d))
    ql = rng.standard_normal((n_layers, B, Hq, d))
    k, v = rng.standard_normal((B * L, Hkv, d)), rng.standard_normal((B * L, Hkv, d))
    res = oracle.shared_index_step(qi, ql, k, v, [0, L, 2 * L], L, 0.25)
    for (b, g), r in res.items():
        for l in range(n_layers):
            for j in range(2):
                h = g * 2 + j
                ref = scipy.special.softmax(0.25 * k[b * L:(b + 1) * L, g] @ ql[l, b, h]) @ v[b * L:(b + 1) * L, g]
                assert np.allclose(r["out"][l, j], ref, rtol=1e-12, atol=1e-13)


def test_shared_index_scores_are_full_dot_and_one_index_per_group():
    rng = np.random.default_rng(15)
    n_layers, B, Hq, Hkv, d, L = 2, 1, 4, 2, 16, 50
    qi = rng.standard_normal((B, Hq, d))
    ql = rng.standard_normal((n_layers, B, Hq, d))
    k, v = rng.standard_normal((L, Hkv, d)), rng.standard_normal((L, Hkv, d))
    res = oracle.shared_index_step(qi, ql, k, v, [0, L], 7, 0.25)
    for g in range(Hkv):
        r = res[(0, g)]
        ref = k[:, g] @ qi[0, 2 * g:2 * g + 2].sum(axis=0)
        assert np.allclose(r["scores"], ref, rtol=1e-12, atol=1e-12)
        assert np.array_equal(r["sel"], np.sort(np.argsort(-ref, kind="stable")[:7]))
        # every layer attends over that same index
        for l in range(n_layers):
            for j in range(2):
                want = oracle.attend(ql[l, 0, 2 * g + j], k[r["sel"], g], v[r["sel"], g], 0.25)
                assert np.allclose(r["out"][l, j], want, rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------------------- appending a token

def test_ring_holds_exactly_the_streaming_positions():
    # the ring of sink + window slots, written position by position, holds the sink plus the
    # recent window: the set the streaming head attends to (brute force over small sizes)
    for sink in range(0, 5):
        for window in range(0, 7):
            for L in range(0, 40):
                held = oracle.ring_contents(L, sink, window)
                kept = held[held >= 0]
                assert len(set(kept.tolist())) == len(kept)  # a slot holds one position, none twice
                assert sorted(kept.tolist()) == oracle.stream_positions(L, sink, window).tolist(), (L, sink, window)
    # hand example: sink 2, window 3, ten tokens: slots hold 0 1 | 8 9 7
    assert oracle.ring_contents(10, 2, 3).tolist() == [0, 1, 8, 9, 7]
    assert oracle.ring_slot(1, 2, 3) == 1 and oracle.ring_slot(2, 2, 3) == 2 and oracle.ring_slot(5, 2, 3) == 2
    assert oracle.ring_slot(7, 4, 0) == -1


def test_bf16_rounding_hand_values_and_library():
    one = 1.0
    assert oracle.to_bf16_bits([one])[0] == 0x3F80
    assert oracle.to_bf16_bits([-2.0])[0] == 0xC000
    assert oracle.to_bf16_bits([1 + 2 ** -8])[0] == 0x3F80       # halfway: ties to the even code
    assert oracle.to_bf16_bits([1 + 3 * 2 ** -8])[0] == 0x3F82   # halfway: ties to the even code
    assert oracle.to_bf16_bits([1 + 2 ** -8 + 2 ** -20])[0] == 0x3F81  # above halfway: up
    assert oracle.to_bf16_bits([0.0])[0] == 0 and oracle.to_bf16_bits([-0.0])[0] == 0x8000
    # the same codes as the library's float32 -> bfloat16 conversion
    import torch

    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.to_bf16_bits(x.astype(np.float64)), lib)
    assert np.array_equal(oracle.bf16_bits_to_f64(lib), torch.from_numpy(lib.view(np.int16)).view(torch.bfloat16)
                          .double().numpy())


def test_append_one_at_a_time_equals_rotating_the_whole_sequence():
    # a key appended when the sequence held p tokens sits at position p: appending L tokens
    # one by one gives the cache that rotating the raw keys at 0 .. L-1 gives
    rng = np.random.default_rng(11)
    d, Hkv, Hq, L, theta = 16, 2, 4, 9, 1e4
    raw_k = rng.standard_normal((L, Hkv, d))
    raw_v = rng.standard_normal((L, Hkv, d))
    raw_q = rng.standard_normal((L, Hq, d))
    for p in range(L):
        qb, kb, vb = oracle.append_token_rows(raw_q[p], raw_k[p], raw_v[p], p, theta)
        for g in range(Hkv):
            whole = oracle.to_bf16_bits(oracle.rope(raw_k[:, g], range(L), theta))
            assert np.array_equal(kb[g], whole[p])
        assert np.array_equal(vb, oracle.to_bf16_bits(raw_v[p]))
        assert np.array_equal(qb, oracle.to_bf16_bits(oracle.rope(raw_q[p], [p] * Hq, theta)))


def test_query_and_key_of_one_token_keep_their_raw_dot():
    # rotated to the same position, a token's q and k have the raw q.k (closed form)
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal((1, 8)), rng.standard_normal((1, 8))
    for p in (0, 1, 17, 4096):
        a = oracle.rope(q, [p], 500.0)[0] @ oracle.rope(k, [p], 500.0)[0]
        assert abs(a - float(q[0] @ k[0])) < 1e-12
        b = oracle.rope(q, [p + 1], 500.0)[0] @ oracle.rope(k, [p], 500.0)[0]
        assert abs(b - float(q[0] @ k[0])) > 1e-6


def test_pack_dominant_row_hand_example():
    k = np.arange(8.0)  # d = 8, chunks 0..3 pair dims (c, c + 4)
    assert oracle.pack_dominant_row(k, [1, 3], 8).tolist() == [1.0, 3.0, 5.0, 7.0, 0, 0, 0, 0]
    assert oracle.pack_dominant_row(k, [0], 2).tolist() == [0.0, 4.0]


# ---------------------------------------------------------------------------- head classifier

def test_proxy_gives_the_singular_values_of_the_full_kernel():
    # Sylvester: the non-zero singular values of M_h = W_K^T W_Q (d_model x d_model) are the
    # square roots of the eigenvalues of the d_head x d_head proxy; checked against a direct
    # SVD of M_h, for square, wide and nearly rank-deficient heads
    rng = np.random.default_rng(21)
    for d_head, d_model in [(6, 40), (8, 8), (3, 50)]:
        for scale in (1.0, 1e-3):
            wq = rng.standard_normal((d_head, d_model))
            wk = rng.standard_normal((d_head, d_model))
            wk[-1] = wk[0] + scale * rng.standard_normal(d_model)  # two close rows when scale is small
            direct = np.linalg.svd(oracle.qk_kernel(wq, wk), compute_uv=False)[:d_head]
            proxy = oracle.proxy_singular_values(wq, wk)
            assert np.allclose(proxy, direct, rtol=1e-7, atol=1e-9 * direct[0]), (d_head, d_model, scale)
            assert oracle.qk_kernel(wq, wk).shape == (d_model, d_model)


def test_effective_rank_hand_examples_and_closed_forms():
    # W_Q = diag(2, 1), W_K = I: M = W_Q, sigma = (2, 1), sigma_hat = (2/3, 1/3)
    wq, wk = np.diag([2.0, 1.0]), np.eye(2)
    assert np.allclose(oracle.proxy_singular_values(wq, wk), [2.0, 1.0])
    er = oracle.effective_rank(oracle.proxy_singular_values(wq, wk))
    assert er == pytest.approx(math.exp(-(2 / 3) * math.log(2 / 3) - (1 / 3) * math.log(1 / 3)), rel=1e-12)
    assert er == pytest.approx(1.8898815748423097, rel=1e-12)
    # one row each: M = k^T q has rank one, sigma = |q| |k| = 5
    assert np.allclose(oracle.proxy_singular_values(np.array([[3.0, 4.0]]), np.array([[1.0, 0.0]])), [5.0])
    assert oracle.effective_rank([5.0]) == 1.0
    # r equal values: ER = r; scale does not matter; zero values are not counted
    for r in (1, 2, 7, 128):
        assert oracle.effective_rank(np.full(r, 3.5)) == pytest.approx(r, rel=1e-12)
    s = np.array([4.0, 2.0, 1.0, 1.0])
    assert oracle.effective_rank(s) == pytest.approx(oracle.effective_rank(1e6 * s), rel=1e-12)
    assert oracle.effective_rank(np.array([4.0, 2.0, 0.0, 0.0])) == pytest.approx(oracle.effective_rank([4.0, 2.0]))
    assert 1.0 < oracle.effective_rank(s) < 4.0


def test_effective_rank_is_blind_to_a_shared_rotation_of_the_model_space():
    # W_Q R and W_K R with R orthogonal (d_model x d_model): M becomes R^T M R, same spectrum
    rng = np.random.default_rng(22)
    wq, wk = rng.standard_normal((5, 30)), rng.standard_normal((5, 30))
    R, _ = np.linalg.qr(rng.standard_normal((30, 30)))
    a = oracle.effective_rank(oracle.proxy_singular_values(wq, wk))
    b = oracle.effective_rank(oracle.proxy_singular_values(wq @ R, wk @ R))
    assert a == pytest.approx(b, rel=1e-10)
    # a head whose query block is low rank has a concentrated spectrum: lower ER
    low = rng.standard_normal((5, 2)) @ rng.standard_normal((2, 30))
    assert oracle.effective_rank(oracle.proxy_singular_values(low, wk)) < a


def test_heads_grouped_by_mean_and_lowest_become_retrieval():
    # two KV groups of two q heads: group 0 = heads 0-1, group 1 = heads 2-3
    rng = np.random.default_rng(23)
    d, dm = 4, 24
    W_Q = rng.standard_normal((4 * d, dm))
    W_K = rng.standard_normal((2 * d, dm))
    er = oracle.head_effective_ranks(W_Q, W_K, 4, 2, d)
    for h in range(4):
        g = h // 2
        assert er[h] == pytest.approx(oracle.effective_rank(np.linalg.svd(
            oracle.qk_kernel(W_Q[h * d:(h + 1) * d], W_K[g * d:(g + 1) * d]), compute_uv=False)[:d]), rel=1e-9)
    grp = oracle.group_effective_ranks(er, 2)
    assert grp.tolist() == pytest.approx([(er[0] + er[1]) / 2, (er[2] + er[3]) / 2])
    assert oracle.group_effective_ranks([1.0, 2.0, 3.0, 6.0, 5.0, 7.0], 2).tolist() == [2.0, 6.0]
    # brute force: the retrieval set is the n lowest, equal values to the lower index
    vals = np.array([3.0, 1.0, 2.0, 1.0, 5.0, 2.0])
    for n in range(0, 7):
        roles = oracle.classify_heads(vals, n)
        chosen = sorted(np.flatnonzero(roles == oracle.ROLE_DENSE).tolist())
        ranked = sorted(range(6), key=lambda g: (vals[g], g))[:n]
        assert chosen == sorted(ranked), n
        assert np.all(roles[roles != oracle.ROLE_DENSE] == oracle.ROLE_STREAM)
    assert oracle.classify_heads(vals, 2).tolist() == [2, 1, 2, 1, 2, 2]


def test_dominant_and_rest_dims_split_every_key():
    # FASA-M keeps the dominant components on the GPU and the rest (with V) on the host: the
    # two sets partition the dims, and a dot product taken part by part is the whole one
    rng = np.random.default_rng(24)
    for d, idom in [(8, [1, 3]), (16, [0, 2, 7]), (128, sorted(rng.choice(64, 16, replace=False)))]:
        dom, rest = oracle.dominant_dims(idom, d), oracle.rest_dims(idom, d)
        assert sorted(dom + rest) == list(range(d)) and not set(dom) & set(rest)
        assert rest == sorted(rest)
        q, k = rng.standard_normal(d), rng.standard_normal(d)
        assert abs(q[dom] @ k[dom] + q[rest] @ k[rest] - q @ k) < 1e-12
    assert oracle.rest_dims([1, 3], 8) == [0, 2, 4, 6]
