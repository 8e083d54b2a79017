"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Tolerances: selected index sets bit-exact except for swaps inside the 1e-4 score
band around the n-th score; scores within 1e-4 of sum |q_c||k_c|; outputs within
2e-3 absolute (unit-variance V).  On caller-given fp32 scores the selection is
compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (OUT_ATOL, SCORE_REL, Dev, check_device, compare_shared_row, compare_sparse_row,
                         compare_window_row, f64, launches_of, row_inputs, run_shared, run_sparse, score_bound,
                         three_kernel_form)
from token_sparse_decode_b200 import binding as B
from workloads import ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, WorkloadSpec, make_workload

pytestmark = pytest.mark.gpu


def spec(**kw):
    base = dict(name="medium", batch=3, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                len_range=(300, 6000), n_dom=16, n_fac_div=8, roles=(ROLE_SPARSE,) * 8,
                planted_frac=0.01, seed=77)
    base.update(kw)
    return WorkloadSpec(**base)


MEDIUM = {
    "gqa4_d128": spec(),
    "gqa7_d128": spec(n_q_heads=28, n_kv_heads=4, roles=(ROLE_SPARSE,) * 4, theta=1e6, seed=78),
    "mha_d64": spec(n_q_heads=4, n_kv_heads=4, head_dim=64, theta=1e4, n_dom=4, roles=(ROLE_SPARSE,) * 4,
                    len_range=(100, 2500), seed=79),
    "gqa16_d64": spec(n_q_heads=32, n_kv_heads=2, head_dim=64, theta=1e4, n_dom=5, roles=(ROLE_SPARSE,) * 2,
                      seed=80),
}


# ------------------------------------------------------------------------------ TIP scores

@pytest.mark.parametrize("name", list(MEDIUM))
@pytest.mark.parametrize("packed", [True, False])
def test_tip_scores_match_oracle(name, packed):
    w = make_workload(MEDIUM[name])
    d = Dev(w)
    k_dom = None
    kv0 = d.kv()
    if packed:
        k_dom = torch.empty((w.spec.n_kv_heads, d.T, B.k_dom_cols(w.spec.n_dom)), dtype=torch.bfloat16,
                            device="cuda")
        B.pack_dominant(kv0, d.idom, w.spec.n_dom, k_dom)
    scores = torch.full((w.spec.n_kv_heads, d.T), float("nan"), device="cuda")
    B.tip_score(d.q, d.kv(k_dom), d.idom, w.spec.n_dom, scores)
    torch.cuda.synchronize()
    check_device()
    got = f64(scores)
    for b in range(w.spec.batch):
        o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
        for g in range(w.spec.n_kv_heads):
            qg, keys, _ = row_inputs(w, b, g)
            idom = w.idom[g].tolist()
            ref = oracle.tip_scores(qg, keys, idom)
            bound = SCORE_REL * score_bound(qg, keys, idom)
            assert np.all(np.abs(got[g, o0:o1] - ref) <= bound), (b, g)


def test_tip_all_chunks_is_full_dot():
    w = make_workload(spec(batch=2, len_range=(1000, 3000)))
    d = Dev(w)
    C = w.spec.head_dim // 2
    all_chunks = torch.arange(C, dtype=torch.int32, device="cuda").repeat(w.spec.n_kv_heads, 1).contiguous()
    scores = torch.empty((w.spec.n_kv_heads, d.T), device="cuda")
    B.tip_score(d.q, d.kv(), all_chunks, C, scores)
    torch.cuda.synchronize()
    got = f64(scores)
    for b in range(2):
        o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
        for g in range(w.spec.n_kv_heads):
            qg, keys, _ = row_inputs(w, b, g)
            ref = keys @ qg.sum(axis=0)
            bound = SCORE_REL * (np.abs(keys) @ np.abs(qg).sum(axis=0))
            assert np.all(np.abs(got[g, o0:o1] - ref) <= bound)


# ------------------------------------------------------------------------------ top-k on given scores

def given_scores(rng, lengths, Hkv, kind):
    T = int(sum(lengths))
    if kind == "normal":
        s = rng.standard_normal((Hkv, T)).astype(np.float32)
    elif kind == "ties":   # few distinct values: ties everywhere, including at the threshold
        s = (np.round(rng.standard_normal((Hkv, T)) * 2) / 2).astype(np.float32)
    elif kind == "zeros":  # -0 and +0 mixed, all equal
        s = np.where(rng.random((Hkv, T)) < 0.5, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
    else:                  # wide dynamic range, negative and positive
        s = (rng.standard_normal((Hkv, T)) * np.exp(rng.uniform(-20, 20, (Hkv, T)))).astype(np.float32)
    return s


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "wide"])
def test_topk_bit_exact_on_given_scores(kind):
    rng = np.random.default_rng(5)
    lengths = [0, 1, 7, 512, 3000, 20000, 65, 131]
    Hkv = 3
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, Hkv, kind)
    nfps = np.array([5, 1, 7, 64, 1000, 2047, 100, 130], dtype=np.int32)
    cap = 2048
    dev = torch.device("cuda")
    k = torch.zeros((int(offs[-1]), Hkv, 64), dtype=torch.bfloat16, device=dev)
    kv = B.make_kv(k, k, torch.from_numpy(offs).to(dev), max(lengths), int(offs[-1]))
    idx = torch.full((len(lengths), Hkv, cap), 12345, dtype=torch.int32, device=dev)
    cnt = torch.full((len(lengths), Hkv), -7, dtype=torch.int32, device=dev)
    B.topk_select(torch.from_numpy(s).to(dev), kv, 0, torch.from_numpy(nfps).to(dev), cap, idx, cnt)
    torch.cuda.synchronize()
    check_device()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b, L in enumerate(lengths):
        for g in range(Hkv):
            row = s[g, offs[b]:offs[b + 1]]
            ref = oracle.select_top(row, int(nfps[b]))
            n = len(ref)
            assert cnt_h[b, g] == n
            assert np.array_equal(idx_h[b, g, :n], ref), (kind, b, g)
            assert np.all(idx_h[b, g, n:] == -1)


def check_topk(s, offs, lengths, nfps, cap, expect_launches, kind):
    Hkv = s.shape[0]
    dev = torch.device("cuda")
    k = torch.zeros((int(offs[-1]), Hkv, 64), dtype=torch.bfloat16, device=dev)
    kv = B.make_kv(k, k, torch.from_numpy(offs).to(dev), max(lengths), int(offs[-1]))
    idx = torch.full((len(lengths), Hkv, cap), 12345, dtype=torch.int32, device=dev)
    cnt = torch.full((len(lengths), Hkv), -7, dtype=torch.int32, device=dev)
    sd, nd = torch.from_numpy(s).to(dev), torch.from_numpy(nfps).to(dev)
    launched = launches_of(lambda: B.topk_select(sd, kv, 0, nd, cap, idx, cnt))
    assert launched == expect_launches
    check_device()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for b, L in enumerate(lengths):
        for g in range(Hkv):
            ref = oracle.select_top(s[g, offs[b]:offs[b + 1]], int(nfps[b]))
            n = len(ref)
            assert cnt_h[b, g] == n, (kind, b, g)
            assert np.array_equal(idx_h[b, g, :n], ref), (kind, b, g)
            assert np.all(idx_h[b, g, n:] == -1), (kind, b, g)


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "wide"])
def test_topk_many_rows(kind):
    # 54 sequences x 3 KV heads = 162 rows, up to 60000 positions: more 8-CTA clusters than
    # one wave holds, so the chunked select runs.  Lengths mix empty, one-token, N_fac >= L
    # and long rows; the ties / zeros kinds leave many keys equal to the threshold, so the
    # lowest positions among them decide.
    rng = np.random.default_rng(15)
    lengths = [0, 1, 3, 700, 24000, 60000] + [int(x) for x in rng.integers(50, 9000, 48)]
    Hkv = 3
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, Hkv, kind)
    nfps = np.array([4, 1, 9, 700, 2048, 1500] + [int(x) for x in rng.integers(1, 2049, 48)], dtype=np.int32)
    check_topk(s, offs, lengths, nfps, 2048,
               {"select_hist_kernel": 1, "select_chunk_kernel": 1, "select_resolve_kernel": 1, "select_write_kernel": 1}, kind)


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "wide"])
def test_topk_rows_in_clusters(kind):
    # 6 sequences x 3 KV heads = 18 rows up to 60000 positions: one wave of 8-CTA clusters,
    # the on-chip select (same score kinds as above)
    rng = np.random.default_rng(18)
    lengths = [0, 3, 700, 24000, 60000, 51234]
    Hkv = 3
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, Hkv, kind)
    nfps = np.array([4, 9, 700, 2048, 1500, 1], dtype=np.int32)
    check_topk(s, offs, lengths, nfps, 2048, {"select_cluster_kernel": 1}, kind)


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "wide"])
def test_topk_long_rows_chunked(kind):
    # a row beyond the row kernel's 256 K positions sends the call to the chunked select
    # (histogram, chunk pass, resolve, ordered write); the ties / zeros kinds put more
    # candidates in the threshold bin than the resolving CTA keeps in shared memory (it then
    # reads them from the list)
    rng = np.random.default_rng(16)
    lengths = [131073, 0, 5, 300000, 2000, 140000]
    Hkv = 2
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, Hkv, kind)
    nfps = np.array([3000, 4, 9, 2048, 2500, 1], dtype=np.int32)
    check_topk(s, offs, lengths, nfps, 3000,
               {"select_hist_kernel": 1, "select_chunk_kernel": 1, "select_resolve_kernel": 1, "select_write_kernel": 1}, kind)


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "wide"])
def test_topk_rows_select_only(kind):
    # rows past the cluster select's 128 K positions, fewer than the SMs: the fused row
    # kernel's select-only mode (keys from the given scores, 16-CTA clusters, 8-bit digits)
    rng = np.random.default_rng(18)
    lengths = [140000, 0, 5, 131073, 131073]
    Hkv = 2
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, Hkv, kind)
    nfps = np.array([2048, 4, 9, 139999, 131072], dtype=np.int32)
    check_topk(s, offs, lengths, nfps, 139999, {"sparse_row_kernel": 1}, kind)


@pytest.mark.parametrize("L", [1, 8191, 8192, 8193, 65536, 131072])
def test_topk_cluster_slice_edges(L):
    # row lengths at the edges of the cluster sizes (8192 positions per CTA): a slice that is
    # full, one position over (the next cluster size), and the largest row one cluster takes
    rng = np.random.default_rng(17 + L)
    lengths = [L, max(1, L // 3)]
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = given_scores(rng, lengths, 2, "normal")
    nfps = np.array([min(2048, max(1, L - 1)), min(2048, max(1, L // 5))], dtype=np.int32)
    check_topk(s, offs, lengths, nfps, 2048, {"select_cluster_kernel": 1}, "normal")


def test_topk_fixed_nfac_and_determinism():
    rng = np.random.default_rng(6)
    lengths = [131072, 4096, 777]
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    s = (np.round(rng.standard_normal((2, int(offs[-1]))) * 8) / 8).astype(np.float32)
    dev = torch.device("cuda")
    k = torch.zeros((int(offs[-1]), 2, 64), dtype=torch.bfloat16, device=dev)
    kv = B.make_kv(k, k, torch.from_numpy(offs).to(dev), max(lengths), int(offs[-1]))
    sd = torch.from_numpy(s).to(dev)
    outs = []
    for _ in range(2):
        idx = torch.empty((3, 2, 2048), dtype=torch.int32, device=dev)
        cnt = torch.empty((3, 2), dtype=torch.int32, device=dev)
        B.topk_select(sd, kv, 2048, None, 2048, idx, cnt)
        torch.cuda.synchronize()
        outs.append((idx.cpu().numpy(), cnt.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    for b in range(3):
        for g in range(2):
            ref = oracle.select_top(s[g, offs[b]:offs[b + 1]], 2048)
            assert np.array_equal(outs[0][0][b, g, :len(ref)], ref)


# ------------------------------------------------------------------------------ sparse decode


@pytest.mark.parametrize("name", list(MEDIUM))
@pytest.mark.parametrize("pack", [True, False])
def test_sparse_decode_matches_oracle(name, pack):
    w = make_workload(MEDIUM[name])
    d = Dev(w)
    step, out = run_sparse(d, pack=pack)
    # a few rows: the whole path in one cluster launch
    assert launches_of(lambda: step(d.q)) == {"sparse_row_kernel": 1}
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = w.spec.group
    stats = {}
    for b in range(w.spec.batch):
        for g in range(w.spec.n_kv_heads):
            n = cnt_h[b, g]
            compare_sparse_row(w, b, g, idx_h[b, g, :n], out_h[b, g * G:(g + 1) * G], stats)
    assert stats["swapped"] <= max(1, stats["rows"] // 10)


def test_sparse_decode_is_deterministic():
    w = make_workload(MEDIUM["gqa4_d128"])
    d = Dev(w)
    step, out = run_sparse(d)
    first = out.clone()
    step(d.q)
    torch.cuda.synchronize()
    assert torch.equal(first, step.out)


# ------------------------------------------------------------------------------ retrieval / streaming heads


@pytest.mark.parametrize("sink,window", [(4, 60), (128, 512), (0, 100), (3000, 4000), (0, 0)])
def test_stream_decode_matches_oracle(sink, window):
    roles = (ROLE_DENSE, ROLE_STREAM, ROLE_STREAM, ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_STREAM, ROLE_STREAM)
    w = make_workload(spec(roles=roles, sink=sink, window=window, len_range=(0, 7000), seed=81))
    d = Dev(w)
    kv = d.kv()
    out = torch.full((w.spec.batch, w.spec.n_q_heads, w.spec.head_dim), 777.0, device="cuda")
    ws = B.workspace(B.stream_decode_workspace_size(kv, w.spec.n_q_heads, roles, sink, window), "cuda")
    B.stream_decode(d.q, kv, roles, sink, window, w.scale, out, ws)
    torch.cuda.synchronize()
    check_device()
    out_h = f64(out)
    G = w.spec.group
    for b in range(w.spec.batch):
        for g, role in enumerate(roles):
            rows = out_h[b, g * G:(g + 1) * G]
            if role == ROLE_SPARSE:
                assert np.all(rows == 777.0)   # not this call's heads: untouched
            else:
                compare_window_row(w, b, g, rows, role, sink, window)


def test_long_dense_rows_merge_in_a_second_launch():
    # DENSE rows of 60-90 K positions split into more than 16 parts: the gather leaves its
    # partials and flash_merge_kernel combines them over many CTAs; the short STREAM rows of
    # the same launch (one or a few splits) go through the same merge
    roles = (ROLE_DENSE, ROLE_STREAM, ROLE_DENSE, ROLE_STREAM)
    w = make_workload(spec(n_q_heads=16, n_kv_heads=4, roles=roles, sink=64, window=512, len_range=(60000, 90000),
                           batch=2, seed=89))
    d = Dev(w)
    kv = d.kv()
    out = torch.full((w.spec.batch, w.spec.n_q_heads, w.spec.head_dim), 777.0, device="cuda")
    ws = B.workspace(B.stream_decode_workspace_size(kv, w.spec.n_q_heads, roles, 64, 512), "cuda")
    launched = launches_of(lambda: B.stream_decode(d.q, kv, roles, 64, 512, w.scale, out, ws))
    assert launched == {"flash_gather_kernel": 1, "flash_merge_kernel": 1}
    check_device()
    out_h = f64(out)
    G = w.spec.group
    for b in range(w.spec.batch):
        for g, role in enumerate(roles):
            compare_window_row(w, b, g, out_h[b, g * G:(g + 1) * G], role, 64, 512)


def test_full_role_split_step_mixed_heads():
    # every row in one wave and window lists no longer than 4 x N_fac: the whole step, window
    # heads included, is one launch of the row kernel
    roles = (ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_SPARSE)
    w = make_workload(spec(n_q_heads=16, n_kv_heads=4, roles=roles, sink=16, window=200, n_fac_div=4, seed=82))
    d = Dev(w)
    step, out = run_sparse(d)
    assert launches_of(lambda: step(d.q)) == {"sparse_row_kernel": 1}
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = w.spec.group
    for b in range(w.spec.batch):
        for g, role in enumerate(roles):
            rows = out_h[b, g * G:(g + 1) * G]
            if role == ROLE_SPARSE:
                compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], rows)
            else:
                compare_window_row(w, b, g, rows, role, w.spec.sink, w.spec.window)


# ------------------------------------------------------------------------------ shared index


@pytest.mark.parametrize("fused", [True, False])
# query rows n_layers * G: 32 and 20 and 18 take two CTAs per row in the three-kernel form (16 rows
# each; the second holds 16, 4 and 2, with a group split across the two for 18), 12 / 8 / 1 one
@pytest.mark.parametrize("n_layers,hq,hkv", [(8, 32, 8), (2, 16, 4), (3, 16, 4), (1, 8, 8), (5, 16, 4), (3, 24, 4)])
def test_shared_index_decode_matches_oracle(n_layers, hq, hkv, fused):
    sp = WorkloadSpec(name="shared", batch=2, n_q_heads=hq, n_kv_heads=hkv, head_dim=128, theta=5e5,
                      len_range=(500, 9000), n_layers=n_layers, topk_shared=700, seed=90 + n_layers)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_shared(d, fused=fused)
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = sp.group
    ref = oracle.shared_index_step(f64(w.q), f64(w.q_layers), f64(w.k), f64(w.v), w.offsets.tolist(), 700,
                                   w.scale)
    for (b, g), r in ref.items():
        sel = idx_h[b, g, :cnt_h[b, g]]
        compare_shared_row(w, b, g, sel, out_h[:, b, g * G:(g + 1) * G], 700)
        if np.array_equal(sel, r["sel"]):  # the stack's own oracle on the same index
            assert np.abs(out_h[:, b, g * G:(g + 1) * G] - r["out"]).max() <= OUT_ATOL


def test_shared_index_reports_out_of_range_positions():
    sp = WorkloadSpec(name="shared", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, theta=1e4,
                      lengths=(300,), n_layers=2, topk_shared=16, seed=3)
    w = make_workload(sp)
    d = Dev(w)
    kv = d.kv()
    idx = torch.arange(16, dtype=torch.int32, device="cuda").repeat(1, 2, 1).contiguous()
    idx[0, 1, 5] = 300            # one past the end of the sequence
    cnt = torch.full((1, 2), 16, dtype=torch.int32, device="cuda")
    out = torch.empty((2, 1, 8, 64), device="cuda")
    ws = B.workspace(B.shared_index_decode_workspace_size(kv, 2, 8, 16), "cuda")
    B.shared_index_decode(d.q_layers, kv, idx, cnt, 16, w.scale, out, ws)
    st, detail = B.device_check()
    assert st == 6 and detail[0] == 1 and detail[3] == 300
    assert B.device_check()[0] == 0   # reading clears the word
    assert torch.isfinite(out).all()


# ------------------------------------------------------------------------------ edge cases


def test_edge_cases_empty_and_short_sequences():
    sp = spec(batch=5, lengths=(0, 1, 2, 64, 65), len_range=None, n_fac_div=0, n_fac=64, n_dom=3,
              planted_frac=0.0, seed=84)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_sparse(d)
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = sp.group
    for b in range(sp.batch):
        for g in range(sp.n_kv_heads):
            n = cnt_h[b, g]
            assert n == min(64, int(w.lengths[b]))
            if w.lengths[b] == 0:
                assert np.all(out_h[b, g * G:(g + 1) * G] == 0.0)
            else:
                compare_sparse_row(w, b, g, idx_h[b, g, :n], out_h[b, g * G:(g + 1) * G])
            assert np.all(idx_h[b, g, n:] == -1)


def test_sparse_decode_long_row_uses_three_kernels():
    # a row longer than one cluster handles (262144 positions) takes the scan / select / attend path
    sp = WorkloadSpec(name="long", batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, theta=1e4, lengths=(300001,),
                      n_dom=6, n_fac=3000, roles=(ROLE_SPARSE,), planted_frac=0.001, seed=85)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_sparse(d)
    assert three_kernel_form(launches_of(lambda: step(d.q)))
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    compare_sparse_row(w, 0, 0, idx_h[0, 0, :cnt_h[0, 0]], out_h[0, 0:2])


def test_sparse_decode_every_token_selected():
    # N_fac >= L on every sequence: focused attention is dense attention
    sp = spec(batch=2, len_range=(50, 900), n_fac_div=0, n_fac=1000, seed=86)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_sparse(d)
    out_h = f64(out)
    G = sp.group
    for b in range(2):
        for g in range(sp.n_kv_heads):
            assert step.count[b, g].item() == w.lengths[b]
            compare_window_row(w, b, g, out_h[b, g * G:(g + 1) * G], ROLE_DENSE, 0, 0)


def test_sparse_decode_many_rows_runs_three_stages():
    # 40 sequences x 8 KV heads = 320 rows: more clusters than one wave holds, so the step
    # runs as scan kernel + select (cluster or chunked) + split-K gather
    sp = spec(batch=40, len_range=(300, 3000), seed=87)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_sparse(d)
    assert three_kernel_form(launches_of(lambda: step(d.q)))
    # the same call with launch events armed: three kernels, in path order, each timed
    rec = B.timed_launches(lambda: B.sparse_decode(d.q, step.kv, step.idom, step.n_dom, step.n_fac,
                                                   step.n_fac_per_seq, step.n_fac_cap, step.roles, step.scale,
                                                   step.out, step.ws, step.idx, step.count))
    torch.cuda.synchronize()
    names = [k for k, _, _ in rec]
    assert names in (["tip_score_kernel", "select_cluster_kernel", "flash_gather_kernel"],
                     ["tip_score_kernel", "select_hist_kernel", "select_chunk_kernel", "select_resolve_kernel",
                      "select_write_kernel", "flash_gather_kernel"])
    assert all(e0.elapsed_time(e1) > 0 for _, e0, e1 in rec)
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = sp.group
    stats = {}
    for b in range(0, sp.batch, 3):
        for g in range(sp.n_kv_heads):
            compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], out_h[b, g * G:(g + 1) * G], stats)
    assert stats["swapped"] <= max(1, stats["rows"] // 10)


def test_shared_index_step_many_rows_runs_three_stages():
    sp = WorkloadSpec(name="shared_many", batch=24, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                      len_range=(500, 9000), n_layers=2, topk_shared=300, seed=88)
    w = make_workload(sp)
    d = Dev(w)
    step, out = run_shared(d, fused=True)
    assert three_kernel_form(launches_of(lambda: step(d.q, d.q_layers)))
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = sp.group
    rows = [(b, g) for b in range(0, 24, 5) for g in range(8)]
    ref = oracle.shared_index_step(f64(w.q), f64(w.q_layers), f64(w.k), f64(w.v), w.offsets.tolist(), 300, w.scale,
                                   rows=rows)
    for (b, g), r in ref.items():
        sel = idx_h[b, g, :cnt_h[b, g]]
        compare_shared_row(w, b, g, sel, out_h[:, b, g * G:(g + 1) * G], 300)
        if np.array_equal(sel, r["sel"]):
            assert np.abs(out_h[:, b, g * G:(g + 1) * G] - r["out"]).max() <= OUT_ATOL


def test_role_split_step_with_long_dense_rows_takes_two_calls():
    # a dense row far longer than a selection keeps the split-K gather: the sparse step, then the window gather
    roles = (ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_SPARSE)
    w = make_workload(spec(n_q_heads=16, n_kv_heads=4, roles=roles, sink=16, window=200, n_fac_div=0, n_fac=48,
                           len_range=(2000, 6000), seed=83))
    d = Dev(w)
    step, out = run_sparse(d)
    launched = launches_of(lambda: step(d.q))
    assert launched.get("flash_gather_kernel", 0) >= 1
    out_h = f64(out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = w.spec.group
    for b in range(w.spec.batch):
        for g, role in enumerate(roles):
            rows = out_h[b, g * G:(g + 1) * G]
            if role == ROLE_SPARSE:
                compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], rows)
            else:
                compare_window_row(w, b, g, rows, role, w.spec.sink, w.spec.window)
