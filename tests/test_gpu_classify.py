"""The AoH head classifier on the GPU against the float64 oracle.

Tolerance: effective ranks within 1e-8 relative.  The GPU forms each Gram matrix on
the fp64 tensor-core path from bf16 weights (exact in fp64, so every product is
exact) and everything after is fp64; it differs from the oracle only in summation
order and in how the eigenvalues are found (Cholesky, congruence and Jacobi against
numpy's eig of C_h), both at the 1e-13 level for these well-conditioned Gram
matrices (numpy's eig of the non-symmetric C_h being the looser of the two), so 1e-8 leaves a wide margin.  (With fp32 accumulation on the bf16 path,
the same tests measured errors up to 2.6e-4 relative on concentrated spectra.)
Roles must match exactly wherever the oracle's group ranks are separated by more
than twice that tolerance at the retrieval boundary (else either order is valid).
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import launches_of
from token_sparse_decode_b200 import binding as B
from workloads import HEAD_WEIGHT_PRESETS, HeadWeightSpec, head_weights

pytestmark = pytest.mark.gpu

ER_REL = 1e-8


def classify_on_gpu(wq, wk, spec, n_retrieval):
    dev = torch.device("cuda")
    er_h = torch.full((spec.n_q_heads,), -1.0, dtype=torch.float64, device=dev)
    er_g = torch.full((spec.n_kv_heads,), -1.0, dtype=torch.float64, device=dev)
    roles = torch.full((spec.n_kv_heads,), 99, dtype=torch.uint8, device=dev)
    ws = B.workspace(B.head_classify_workspace_size(spec.d_model, spec.n_q_heads, spec.n_kv_heads, spec.head_dim), dev)
    wq_d, wk_d = wq.to(dev), wk.to(dev)
    launched = launches_of(lambda: B.head_classify(wq_d, wk_d, spec.n_q_heads, spec.n_kv_heads, spec.head_dim,
                                                   n_retrieval, er_h, er_g, roles, ws))
    assert launched == {"gram_kernel": 1, "gram_reduce_kernel": 1, "spectrum_kernel": 1, "group_roles_kernel": 1}
    return er_h.cpu().numpy(), er_g.cpu().numpy(), roles.cpu().numpy()


def check_against_oracle(spec, wq, wk, n_retrieval):
    er_h, er_g, roles = classify_on_gpu(wq, wk, spec, n_retrieval)
    assert B.device_check()[0] == 0
    ref_h = oracle.head_effective_ranks(wq.double().numpy(), wk.double().numpy(), spec.n_q_heads, spec.n_kv_heads,
                                        spec.head_dim)
    ref_g = oracle.group_effective_ranks(ref_h, spec.n_kv_heads)
    assert np.all(np.abs(er_h - ref_h) <= ER_REL * ref_h), np.abs(er_h / ref_h - 1).max()
    assert np.all(np.abs(er_g - ref_g) <= ER_REL * ref_g)
    ref_roles = oracle.classify_heads(ref_g, n_retrieval)
    srt = np.sort(ref_g)
    if 0 < n_retrieval < spec.n_kv_heads and srt[n_retrieval] - srt[n_retrieval - 1] <= 2 * ER_REL * srt[n_retrieval]:
        # a near tie at the boundary: the GPU's roles follow its own ranks
        assert np.array_equal(roles, oracle.classify_heads(er_g, n_retrieval))
    else:
        assert np.array_equal(roles, ref_roles), (roles, ref_roles)
    return er_h, er_g, roles


@pytest.mark.parametrize("name", sorted(HEAD_WEIGHT_PRESETS))
def test_head_classifier_matches_oracle(name):
    spec = HEAD_WEIGHT_PRESETS[name]
    wq, wk, ranks = head_weights(spec)
    er_h, er_g, roles = check_against_oracle(spec, wq, wk, spec.n_retrieval)
    # the structured (low-rank) groups are the retrieval heads of these weights
    assert set(np.flatnonzero(roles == 1)) == set(np.flatnonzero(ranks > 0))
    # the same call twice: the same bits (fixed summation orders)
    again = classify_on_gpu(wq, wk, spec, spec.n_retrieval)
    assert np.array_equal(again[0], er_h) and np.array_equal(again[1], er_g) and np.array_equal(again[2], roles)


@pytest.mark.parametrize("n_retrieval", [0, 1, 3, 6])
def test_head_classifier_every_retrieval_count(n_retrieval):
    spec = HeadWeightSpec(name="mixed", n_q_heads=12, n_kv_heads=6, head_dim=128, d_model=1024,
                          ranks=(1, 5, 0, 20, 0, 40), seed=608)
    wq, wk, _ = head_weights(spec)
    check_against_oracle(spec, wq, wk, n_retrieval)


def test_head_classifier_short_model_dimension():
    # d_model 192: one split of 192 columns (a multiple of 64 that is not one of 512)
    spec = HeadWeightSpec(name="short", n_q_heads=4, n_kv_heads=2, head_dim=64, d_model=192, ranks=(2, 0), seed=609)
    wq, wk, _ = head_weights(spec)
    check_against_oracle(spec, wq, wk, 1)


def test_key_block_without_full_rank_is_reported():
    spec = HeadWeightSpec(name="zero_row", n_q_heads=4, n_kv_heads=2, head_dim=64, d_model=256, ranks=(0, 0),
                          seed=610)
    wq, wk, _ = head_weights(spec)
    wk[64 + 5] = 0  # a zero row in KV head 1's block: its Gram matrix is singular
    er_h, er_g, roles = classify_on_gpu(wq, wk, spec, 1)
    st, detail = B.device_check()
    assert st == 6 and detail[0] == 5 and detail[1] in (2, 3)
    assert np.all(np.isfinite(er_h[:2])) and np.all(np.isnan(er_h[2:]))
    ref = oracle.head_effective_ranks(wq.double().numpy(), wk.double().numpy(), 4, 2, 64)
    assert np.all(np.abs(er_h[:2] - ref[:2]) <= ER_REL * ref[:2])
