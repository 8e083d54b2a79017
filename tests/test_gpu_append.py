"""The append path against the oracle, one decode step at a time.

Every step draws a new token per sequence (its raw q, k, v), appends it through
aoh_kv_append (rotation to its position, K / V rows into the linear cache for the
retrieval heads and into the ring for the streaming heads, the packed dominant row)
and decodes over positions 0 .. p.  Checked after every step:
  * cache bytes: the rotated query, the K / V rows and the packed dominant row equal
    the oracle's bf16 codes bit for bit (a code may differ only where the oracle's
    float64 value lies within 1e-12 of a rounding boundary, which the two sides'
    double-precision sines may then round apart);
  * lengths advanced by one;
  * outputs: SPARSE heads' selection within the tie band of the oracle's scores and
    output within 2e-3; DENSE and STREAM heads within 2e-3 of the oracle over
    [0, p] and over the sink + window, read from the ring.
Unwritten positions of the caches hold NaN, so a read of any of them would show.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (OUT_ATOL, Dev, check_device, check_selection, compare_shared_row, compare_sparse_row,
                         compare_window_row, f64, launches_of, output_tolerance, score_floor, three_kernel_form)
from token_sparse_decode_b200 import binding as B
from token_sparse_decode_b200.step import AppendDecodeStep, SharedIndexStep, SparseDecodeStep
from workloads import ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, WorkloadSpec, make_workload, token_draws

pytestmark = pytest.mark.gpu

def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def assert_codes(gpu_bits, ref_bits, exact_values=None, what=""):
    """Equal bf16 codes; a mismatch is allowed only on a rounding boundary of the exact value."""
    gpu_bits, ref_bits = np.asarray(gpu_bits), np.asarray(ref_bits)
    bad = gpu_bits != ref_bits
    if not bad.any():
        return 0
    assert exact_values is not None, f"{what}: {int(bad.sum())} codes differ"
    x = np.asarray(exact_values, dtype=np.float64)[bad]
    lo = oracle.to_bf16_bits(x * (1 - 1e-12))
    hi = oracle.to_bf16_bits(x * (1 + 1e-12))
    assert np.all(lo != hi), f"{what}: {int(bad.sum())} codes differ away from a rounding boundary"
    return int(bad.sum())


class OracleCaches:
    """The oracle's view: every (sequence, KV head)'s key and value codes, position by position."""

    def __init__(self, B_, Hkv):
        self.k = {(b, g): [] for b in range(B_) for g in range(Hkv)}
        self.v = {(b, g): [] for b in range(B_) for g in range(Hkv)}

    def rows(self, b, g):
        k = oracle.bf16_bits_to_f64(np.array(self.k[(b, g)], dtype=np.uint16).reshape(-1, self.d))
        v = oracle.bf16_bits_to_f64(np.array(self.v[(b, g)], dtype=np.uint16).reshape(-1, self.d))
        return k, v


def prefix(step: AppendDecodeStep, orc: OracleCaches, L0, seed):
    """Positions 0 .. L0_b - 1 of every sequence, written into both sides' caches by the test."""
    d, theta = step.d, step.theta
    for b, Lb in enumerate(L0):
        r = np.random.default_rng([seed, b])
        raw_k = r.standard_normal((Lb, step.Hkv, d))
        raw_v = r.standard_normal((Lb, step.Hkv, d))
        o = int(step.offsets[b])
        for g in range(step.Hkv):
            kb = oracle.to_bf16_bits(oracle.rope(raw_k[:, g], range(Lb), theta)) if Lb else np.zeros((0, d), np.uint16)
            vb = oracle.to_bf16_bits(raw_v[:, g]) if Lb else np.zeros((0, d), np.uint16)
            orc.k[(b, g)] = list(kb)
            orc.v[(b, g)] = list(vb)
            if Lb == 0:
                continue
            if step.lin_slot[g] != B.NO_SLOT:
                s = step.lin_slot[g]
                step.k[o:o + Lb, s] = to_dev_bf16(kb)
                step.v[o:o + Lb, s] = to_dev_bf16(vb)
            if step.ring_slot[g] != B.NO_SLOT:
                s, ro = step.ring_slot[g], b * (step.sink + step.window)
                for j, pos in enumerate(oracle.ring_contents(Lb, step.sink, step.window)):
                    if pos >= 0:
                        step.rk[ro + j, s] = to_dev_bf16(kb[pos])
                        step.rv[ro + j, s] = to_dev_bf16(vb[pos])
    step.lengths.copy_(torch.tensor(L0, dtype=torch.int32))
    if step.k_dom is not None:
        B.pack_dominant(step.kv, step.idom, step.n_dom, step.k_dom)


def run_session(d, roles, L0, capacity_extra, steps, sink, window, n_fac, seed):
    G = 4 if d == 128 else 2
    Hkv = len(roles)
    Hq = G * Hkv
    C = d // 2
    theta = 5e5 if d == 128 else 1e4
    rng = np.random.default_rng(seed)
    n_dom = 16 if d == 128 else 5
    idom = np.stack([np.sort(rng.choice(C, n_dom, replace=False)) for _ in range(Hkv)]).astype(np.int32)
    Bn = len(L0)
    step = AppendDecodeStep(Bn, Hq, Hkv, d, theta, roles, [L + capacity_extra for L in L0], sink, window,
                            1.0 / np.sqrt(d), idom=torch.from_numpy(idom).cuda(), n_fac=n_fac)
    # every position not yet written reads as NaN
    for t in (step.k, step.v) + ((step.rk, step.rv) if step.ring is not None else ()):
        t.fill_(float("nan"))
    orc = OracleCaches(Bn, Hkv)
    orc.d = d
    prefix(step, orc, L0, seed)
    torch.cuda.synchronize()
    L = list(L0)
    cols = B.k_dom_cols(n_dom)
    flips = 0
    for t in range(steps):
        qn, kn, vn = token_draws(seed, t, Bn, Hq, Hkv, d)
        launched = launches_of(lambda: step(qn.cuda(), kn.cuda(), vn.cuda()))
        assert launched.get("kv_append_kernel") == 1
        check_device()
        assert step.lengths.cpu().tolist() == [x + 1 for x in L]
        q_rot = bits_of(step.q_rot)
        k_lin, v_lin = bits_of(step.k), bits_of(step.v)
        k_dom = bits_of(step.k_dom) if step.k_dom is not None else None
        k_ring = bits_of(step.rk) if step.ring is not None else None
        v_ring = bits_of(step.rv) if step.ring is not None else None
        for b in range(Bn):
            p = L[b]
            qr, kr, vr = (x[b].double().numpy() for x in (qn, kn, vn))
            qb, kb, vb = oracle.append_token_rows(qr, kr, vr, p, theta)
            q_exact = oracle.rope(qr, [p] * Hq, theta)
            k_exact = oracle.rope(kr, [p] * Hkv, theta)
            flips += assert_codes(q_rot[b], qb, q_exact, f"q_rot[{b}]")
            o = int(step.offsets[b])
            for g in range(Hkv):
                if step.lin_slot[g] != B.NO_SLOT:
                    s = step.lin_slot[g]
                    flips += assert_codes(k_lin[o + p, s], kb[g], k_exact[g], f"k[{b},{g}]")
                    assert_codes(v_lin[o + p, s], vb[g], what=f"v[{b},{g}]")
                    if k_dom is not None:
                        want = oracle.pack_dominant_row(kb[g], idom[g], cols)
                        exact = oracle.pack_dominant_row(k_exact[g], idom[g], cols)
                        flips += assert_codes(k_dom[s, o + p], want, exact, f"k_dom[{b},{g}]")
                if step.ring_slot[g] != B.NO_SLOT:
                    slot = oracle.ring_slot(p, sink, window)
                    if slot >= 0:
                        ro, s = b * (sink + window), step.ring_slot[g]
                        flips += assert_codes(k_ring[ro + slot, s], kb[g], k_exact[g], f"ring k[{b},{g}]")
                        assert_codes(v_ring[ro + slot, s], vb[g], what=f"ring v[{b},{g}]")
                orc.k[(b, g)].append(kb[g])
                orc.v[(b, g)].append(vb[g])
            L[b] += 1
            # the outputs of every head of this sequence, over positions 0 .. p
            out = f64(step.out[b])
            qf = oracle.bf16_bits_to_f64(qb)
            for g, role in enumerate(roles):
                keys, vals = orc.rows(b, g)
                qg = qf[g * G:(g + 1) * G]
                got = out[g * G:(g + 1) * G]
                if role == ROLE_SPARSE:
                    s = oracle.tip_scores(qg, keys, idom[g])
                    n = min(n_fac, L[b])
                    sel = step.idx[b, g, :int(step.count[b, g])].cpu().numpy()
                    beta = check_selection(sel, s, n, score_floor(qg, keys, idom[g]))
                    ref_sel = oracle.select_top(s, n)
                    ref = oracle.focused_attention(qg, keys, vals, ref_sel, step.scale)
                    tol = output_tolerance(sel, ref_sel, qg, keys, vals, s, n, step.scale, beta)
                else:
                    pos = (oracle.dense_positions(L[b]) if role == ROLE_DENSE
                           else oracle.stream_positions(L[b], sink, window))
                    ref = oracle.focused_attention(qg, keys, vals, pos, step.scale)
                    tol = OUT_ATOL
                assert np.isfinite(got).all(), (t, b, g)
                assert np.abs(got - ref).max() <= tol, (t, b, g, role, np.abs(got - ref).max())
    return flips


@pytest.mark.parametrize("d", [64, 128])
def test_append_then_decode_step_by_step(d):
    roles = (ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_SPARSE, ROLE_STREAM)
    flips = run_session(d, roles, L0=[0, 37, 150], capacity_extra=14, steps=12, sink=8, window=40, n_fac=24,
                        seed=900 + d)
    assert flips <= 2  # codes decided apart on a rounding boundary: expected almost never


def test_append_streaming_heads_only_and_long_wrap():
    # every head streams: no linear cache at all; a 300-token prefix wraps the window many times
    roles = (ROLE_STREAM,) * 4
    run_session(128, roles, L0=[300, 5], capacity_extra=0, steps=9, sink=4, window=16, n_fac=0, seed=931)


def test_append_to_a_full_region_is_refused_on_the_device():
    Hkv, Hq, d = 2, 4, 64
    step = AppendDecodeStep(2, Hq, Hkv, d, 1e4, (ROLE_DENSE, ROLE_DENSE), [2, 5], 0, 0, 0.125)
    for t in range(3):
        qn, kn, vn = token_draws(7, t, 2, Hq, Hkv, d)
        step.append(qn.cuda(), kn.cuda(), vn.cuda())
        torch.cuda.synchronize()
        st, detail = B.device_check()
        if t < 2:
            assert st == 0
        else:  # sequence 0 is full after two tokens: its third is refused, sequence 1 takes its own
            assert st == 6 and detail[0] == 4 and detail[1] == 0 and detail[2] == 2 and detail[3] == 2
    assert step.lengths.cpu().tolist() == [2, 3]


# ------------------------------------------------------------------------------ decoding with lengths

def capacity_layout(w, extra_seed):
    """The workload's cache in per-sequence regions with unused room (NaN) past each length."""
    rng = np.random.default_rng(extra_seed)
    L = w.lengths.astype(np.int64)
    cap = L + rng.integers(0, 700, len(L))
    offs = np.concatenate([[0], np.cumsum(cap)]).astype(np.int32)
    T = int(offs[-1])
    Hkv, d = w.spec.n_kv_heads, w.spec.head_dim
    k = torch.full((T, Hkv, d), float("nan"), dtype=torch.bfloat16)
    v = torch.full((T, Hkv, d), float("nan"), dtype=torch.bfloat16)
    for b in range(len(L)):
        o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
        k[offs[b]:offs[b] + o1 - o0] = w.k[o0:o1]
        v[offs[b]:offs[b] + o1 - o0] = w.v[o0:o1]
    return k.cuda(), v.cuda(), torch.from_numpy(offs).cuda(), torch.from_numpy(L.astype(np.int32)).cuda(), T, int(cap.max())


@pytest.mark.parametrize("batch", [3, 40])
def test_decode_reads_only_up_to_each_length(batch):
    roles = (ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_SPARSE, ROLE_SPARSE, ROLE_STREAM, ROLE_SPARSE, ROLE_SPARSE)
    sp = WorkloadSpec(name="lengths", batch=batch, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                      len_range=(100, 4000), n_dom=16, n_fac_div=8, roles=roles, sink=32, window=300,
                      planted_frac=0.01, seed=940 + batch)
    w = make_workload(sp)
    k, v, offs, lengths, T, max_cap = capacity_layout(w, 941)
    d = Dev(w)
    for pack in (True, False):
        k_dom = None
        if pack:
            k_dom = torch.empty((8, T, B.k_dom_cols(16)), dtype=torch.bfloat16, device="cuda")
            B.pack_dominant(B.make_kv(k, v, offs, max_cap, T), d.idom, 16, k_dom)
        kv = B.make_kv(k, v, offs, max_cap, T, k_dom, lengths)
        nfac = int(w.n_fac_per_seq.max())
        out = torch.full((batch, 32, 128), 9.0, device="cuda")
        idx = torch.empty((batch, 8, nfac), dtype=torch.int32, device="cuda")
        cnt = torch.empty((batch, 8), dtype=torch.int32, device="cuda")
        ws = B.workspace(B.sparse_decode_workspace_size(kv, 32, nfac), "cuda")
        run = launches_of(lambda: B.sparse_decode(d.q, kv, d.idom, 16, nfac, d.n_fac_per_seq, nfac, list(roles),
                                                  w.scale, out, ws, idx, cnt))
        assert (run == {"sparse_row_kernel": 1}) if batch == 3 else three_kernel_form(run)
        ws2 = B.workspace(B.stream_decode_workspace_size(kv, 32, list(roles), sp.sink, sp.window), "cuda")
        B.stream_decode(d.q, kv, list(roles), sp.sink, sp.window, w.scale, out, ws2)
        torch.cuda.synchronize()
        check_device()
        out_h, idx_h, cnt_h = f64(out), idx.cpu().numpy(), cnt.cpu().numpy()
        for b in range(0, batch, 1 if batch == 3 else 6):
            for g, role in enumerate(roles):
                o = out_h[b, g * 4:(g + 1) * 4]
                if role == ROLE_SPARSE:
                    compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], o)
                else:
                    compare_window_row(w, b, g, o, role, sp.sink, sp.window)


@pytest.mark.parametrize("batch", [2, 24])
def test_shared_index_step_reads_only_up_to_each_length(batch):
    sp = WorkloadSpec(name="lengths_shared", batch=batch, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                      len_range=(500, 6000), n_layers=2, topk_shared=300, seed=950 + batch)
    w = make_workload(sp)
    k, v, offs, lengths, T, max_cap = capacity_layout(w, 951)
    d = Dev(w)
    step = SharedIndexStep(k, v, offs, max_cap, T, 2, 32, 300, w.scale)
    step.kv = B.make_kv(k, v, offs, max_cap, T, None, lengths)
    step(d.q, d.q_layers)
    torch.cuda.synchronize()
    check_device()
    out_h, idx_h, cnt_h = f64(step.out), step.idx.cpu().numpy(), step.count.cpu().numpy()
    for b in range(0, batch, 1 if batch == 2 else 5):
        for g in range(8):
            compare_shared_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], out_h[:, b, g * 4:(g + 1) * 4], 300)
