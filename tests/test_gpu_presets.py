"""Parity at the five workloads' full sizes, in the launch configuration bench.py
times (SparseDecodeStep / SharedIndexStep), on every row or on a seeded sample of
rows that the oracle computes one by one."""

import numpy as np
import pytest
import torch

from gpu_helpers import (Dev, compare_shared_row, compare_sparse_row, compare_window_row, f64, launches_of, run_shared,
                         run_sparse)
from workloads import ROLE_SPARSE, make_workload, preset

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_rows(w, n, seed=0):
    rows = [(b, g) for b in range(w.spec.batch) for g in range(w.spec.n_kv_heads)]
    if len(rows) <= n:
        return rows
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(rows), n, replace=False)
    return [rows[i] for i in sorted(pick)]


def check_role_split(name, n_rows, pack=True):
    w = make_workload(preset(name))
    d = Dev(w)
    step, out = run_sparse(d, pack=pack)
    out_h = f64(out)
    G = w.spec.group
    stats = {}
    idx_h = step.idx.cpu().numpy() if step.has_sparse else None
    cnt_h = step.count.cpu().numpy() if step.has_sparse else None
    for b, g in sample_rows(w, n_rows):
        rows = out_h[b, g * G:(g + 1) * G]
        if int(w.roles[g]) == ROLE_SPARSE:
            compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], rows, stats)
        else:
            compare_window_row(w, b, g, rows, int(w.roles[g]), w.spec.sink, w.spec.window)
    if stats:
        assert stats["swapped"] <= max(1, stats["rows"] // 10)
    del d, step, out
    torch.cuda.empty_cache()


def test_tiny_mixed_d64_L512_all_rows():
    check_role_split("tiny_mixed_d64_L512", 10 ** 9)


def test_tiny_mixed_step_is_one_launch():
    # 2 sparse + 2 streaming heads of a 512-token sequence: one row-kernel launch, one CTA a row
    w = make_workload(preset("tiny_mixed_d64_L512"))
    d = Dev(w)
    step, _ = run_sparse(d)
    assert launches_of(lambda: step(d.q)) == {"sparse_row_kernel": 1}


def test_llama8b_gqa4_L32k_all_rows():
    check_role_split("llama8b_gqa4_L32k", 10 ** 9)


def test_llama8b_gqa4_L32k_in_place_scan_all_rows():
    # no packed dominant columns: the scan reads the 16-byte segments of K that hold them
    check_role_split("llama8b_gqa4_L32k", 10 ** 9, pack=False)


def test_aoh_roles_L128k_all_rows():
    check_role_split("aoh_roles_L128k", 10 ** 9)


def test_fasa_serving_ragged_b64_sampled_rows():
    check_role_split("fasa_serving_ragged_b64", 48)


def test_clsa_shared_L128k_all_rows():
    w = make_workload(preset("clsa_shared_L128k"))
    d = Dev(w)
    step, out = run_shared(d)
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = w.spec.group
    for b, g in sample_rows(w, 10 ** 9):
        compare_shared_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], out_h[:, b, g * G:(g + 1) * G], w.spec.topk_shared)
