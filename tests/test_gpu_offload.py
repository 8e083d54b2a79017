"""FASA-M (host offload) against the oracle and against the resident path.

The host parts written by aoh_offload_split must be the cache's non-dominant key
dims (ascending, zero-padded) and its values, bit for bit.  A decode step on the
offloaded cache must select exactly what the resident step selects from the same
dominant columns (the same scan arithmetic), within the tie band of the oracle's
scores, and give outputs within 2e-3 of the oracle.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import Dev, check_device, compare_sparse_row, f64, launches_of, run_sparse
from token_sparse_decode_b200 import binding as B
from token_sparse_decode_b200.step import OffloadDecodeStep
from workloads import ROLE_SPARSE, WorkloadSpec, make_workload

pytestmark = pytest.mark.gpu


def bits(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


CASES = {
    "gqa4_d128": WorkloadSpec(name="off128", batch=3, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                              len_range=(300, 6000), n_dom=16, n_fac_div=8, roles=(ROLE_SPARSE,) * 8,
                              planted_frac=0.01, seed=960),
    "mha_d64": WorkloadSpec(name="off64", batch=4, n_q_heads=4, n_kv_heads=4, head_dim=64, theta=1e4,
                            len_range=(50, 2500), n_dom=4, n_fac_div=8, roles=(ROLE_SPARSE,) * 4, seed=961),
    "many_rows": WorkloadSpec(name="offmany", batch=40, n_q_heads=16, n_kv_heads=4, head_dim=128, theta=1e6,
                              len_range=(100, 3000), n_dom=12, n_fac=256, roles=(ROLE_SPARSE,) * 4, seed=962),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_offload_decode_matches_oracle_and_resident_path(name):
    w = make_workload(CASES[name])
    d = Dev(w)
    nfac = int(w.n_fac_per_seq.max())
    step = OffloadDecodeStep(d.k, d.v, d.offsets, d.max_len, d.T, w.spec.n_q_heads, d.idom, w.scale, n_fac=nfac,
                             n_fac_per_seq=d.n_fac_per_seq, n_fac_cap=nfac)
    check_device()
    # the host parts, bit for bit
    kr, vh = bits(step.k_rest), bits(step.v_host)
    kb, vb = bits(w.k), bits(w.v)
    for g in range(w.spec.n_kv_heads):
        rest = oracle.rest_dims(w.idom[g].tolist(), w.spec.head_dim)
        assert np.array_equal(kr[g, :, :len(rest)], kb[:, g, rest])
        assert np.all(kr[g, :, len(rest):] == 0)
        assert np.array_equal(vh[g], vb[:, g])
    launched = launches_of(lambda: step(d.q))
    assert launched.get("offload_stage_kernel") == 1 and launched.get("tip_score_kernel") == 1
    assert launched.get("flash_gather_kernel") == 1
    check_device()
    out_h = f64(step.out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    res, res_out = run_sparse(d)
    r_idx, r_cnt = res.idx.cpu().numpy(), res.count.cpu().numpy()
    G = w.spec.group
    for b in range(0, w.spec.batch, 1 if w.spec.batch < 10 else 5):
        for g in range(w.spec.n_kv_heads):
            n = cnt_h[b, g]
            assert n == r_cnt[b, g] and np.array_equal(idx_h[b, g, :n], r_idx[b, g, :n])
            compare_sparse_row(w, b, g, idx_h[b, g, :n], out_h[b, g * G:(g + 1) * G])
    assert np.abs(out_h - f64(res_out)).max() <= 1e-4  # the same selection: only summation order differs


def test_pageable_host_memory_is_refused():
    w = make_workload(CASES["mha_d64"])
    d = Dev(w)
    step = OffloadDecodeStep(d.k, d.v, d.offsets, d.max_len, d.T, 4, d.idom, w.scale, n_fac=64, n_fac_cap=64)
    pageable = torch.empty_like(step.v_host, pin_memory=False)
    oc = B.OffloadCache.from_buffer_copy(step.oc)
    oc.v = pageable.data_ptr()
    with pytest.raises(B.AohError) as e:
        B.offload_decode(d.q, oc, d.idom, 4, 64, None, 64, w.scale, step.out, step.ws)
    assert e.value.status == 1
    assert B.device_check()[0] == 0
