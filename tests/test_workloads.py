"""The seeded input generator: determinism, shapes, the recipe's structure."""

import math

import numpy as np
import torch

import oracle
from workloads import PRESETS, ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, WorkloadSpec, make_workload, preset
from workloads.synth import key_block_raw, query_raw


def small_spec(**kw):
    base = dict(name="small", batch=3, n_q_heads=8, n_kv_heads=2, head_dim=64, theta=1e4,
                len_range=(40, 300), n_dom=4, n_fac=32, planted_frac=0.05, seed=9)
    base.update(kw)
    return WorkloadSpec(**base)


def test_deterministic_and_shaped():
    s = small_spec()
    a, b = make_workload(s), make_workload(s, threads=1)
    assert torch.equal(a.k.view(torch.int16), b.k.view(torch.int16))
    assert torch.equal(a.v.view(torch.int16), b.v.view(torch.int16))
    assert torch.equal(a.q.view(torch.int16), b.q.view(torch.int16))
    T = int(a.lengths.sum())
    assert a.k.shape == (T, 2, 64) and a.v.shape == (T, 2, 64) and a.q.shape == (3, 8, 64)
    assert a.offsets.dtype == torch.int32 and a.offsets[-1].item() == T
    assert np.all((a.lengths >= 40) & (a.lengths <= 300))
    assert a.idom.shape == (2, 4) and torch.all(a.idom[:, 1:] > a.idom[:, :-1])
    c = make_workload(small_spec(seed=10))
    assert not torch.equal(a.q.view(torch.int16), c.q.view(torch.int16))


def test_keys_are_rotated_raw_draws_at_their_positions():
    s = small_spec(planted_frac=0.0)
    w = make_workload(s)
    b, g = 1, 1
    raw = key_block_raw(s, b, g).astype(np.float64)
    L = int(w.lengths[b])
    want = oracle.rope(raw, range(L), s.theta)
    o = int(w.offsets[b])
    got = w.k[o:o + L, g].double().numpy()
    # bf16 rounding of the rotated float32 values: relative 2^-8
    assert np.allclose(got, want, rtol=2 ** -8, atol=1e-6)
    qraw = query_raw(s, b, 5).astype(np.float64)
    qwant = oracle.rope(qraw[None, :], [L], s.theta)[0]
    assert np.allclose(w.q[b, 5].double().numpy(), qwant, rtol=2 ** -8, atol=1e-6)


def test_planted_keys_are_boosted_on_dominant_chunks():
    s = small_spec(planted_frac=0.05, planted_gain=4.0, theta=1e4)
    w = make_workload(s)
    for (b, g), toks in w.planted.items():
        L = int(w.lengths[b])
        assert len(toks) == math.ceil(0.05 * L)
        raw = key_block_raw(s, b, g)
        C = s.head_dim // 2
        dims = oracle.dominant_dims(w.idom[g].tolist(), s.head_dim)
        # boosted rows have a larger norm on the dominant dims than the rest on average
        if len(toks):
            boosted = np.abs(raw[toks][:, dims]).mean()
            rest = np.abs(np.delete(raw, toks, axis=0)[:, dims]).mean()
            assert boosted > 1.4 * rest


def test_presets_structure():
    p = PRESETS
    assert p["llama8b_gqa4_L32k"].group == 4 and p["fasa_serving_ragged_b64"].group == 7
    roles = make_workload(preset("tiny_mixed_d64_L512")).roles.tolist()
    assert roles == [ROLE_SPARSE, ROLE_SPARSE, ROLE_STREAM, ROLE_STREAM]
    # the role draw of the head-role split: exactly 2 dense groups of 8, seeded
    from workloads.synth import _draw_roles, _draw_lengths, _n_fac
    r = _draw_roles(p["aoh_roles_L128k"])
    assert (r == ROLE_DENSE).sum() == 2 and (r == ROLE_STREAM).sum() == 6
    spec5 = p["fasa_serving_ragged_b64"]
    L = _draw_lengths(spec5)
    assert L.shape == (64,) and L.min() >= 4096 and L.max() <= 65536
    assert np.array_equal(_n_fac(spec5, L), [-(-int(x) // 8) for x in L])
