"""Parity at the five workloads' full sizes, in the launch configuration bench.py
times (SparseDecodeStep / SharedIndexStep), on every row or on a seeded sample of
rows that the oracle computes one by one."""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (OUT_ATOL, Dev, band_swap_bound, compare_sparse_row, compare_window_row, f64, row_inputs,
                         run_shared, run_sparse)
from workloads import ROLE_SPARSE, make_workload, preset

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_rows(w, n, seed=0):
    rows = [(b, g) for b in range(w.spec.batch) for g in range(w.spec.n_kv_heads)]
    if len(rows) <= n:
        return rows
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(rows), n, replace=False)
    return [rows[i] for i in sorted(pick)]


def check_role_split(name, n_rows):
    w = make_workload(preset(name))
    d = Dev(w)
    step, out = run_sparse(d)
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


def test_llama8b_gqa4_L32k_all_rows():
    check_role_split("llama8b_gqa4_L32k", 10 ** 9)


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
    k = w.spec.topk_shared
    for b, g in sample_rows(w, 10 ** 9):
        o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
        qg, keys, values = row_inputs(w, b, g)
        qi = f64(w.q[b, g * G:(g + 1) * G])
        s = oracle.tip_scores(qi, keys, range(w.spec.head_dim // 2))
        n = min(k, o1 - o0)
        sel = idx_h[b, g, :cnt_h[b, g]]
        ok, msg = oracle.tie_band_check(sel, s, n)
        assert ok, msg
        ref_sel = oracle.select_top(s, n)
        tol = OUT_ATOL
        for l in range(w.spec.n_layers):
            ql = f64(w.q_layers[l, b, g * G:(g + 1) * G])
            ref = oracle.focused_attention(ql, keys, values, ref_sel, w.scale)
            t = tol if np.array_equal(sel, ref_sel) else tol + band_swap_bound(ql, keys, values, s, n, w.scale)
            err = np.abs(out_h[l, b, g * G:(g + 1) * G] - ref).max()
            assert err <= t, (b, g, l, err)
