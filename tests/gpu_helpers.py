"""Shared helpers of the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, compare with the float64 oracle on the same inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from token_sparse_decode_b200 import binding as B
from token_sparse_decode_b200.step import SharedIndexStep, SparseDecodeStep

OUT_ATOL = 2e-3        # outputs, absolute, unit-variance V
SCORE_REL = 1e-4       # scores, relative to sum |q_c| |k_c| over the scored dims
BAND_REL = 1e-4        # top-k tie band, relative to the n-th score


class Dev:
    """A Workload's tensors on the GPU."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.k = w.k.to(device)
        self.v = w.v.to(device)
        self.q = w.q.to(device)
        self.q_layers = None if w.q_layers is None else w.q_layers.to(device)
        self.offsets = w.offsets.to(device)
        self.idom = None if w.idom is None else w.idom.to(device)
        self.n_fac_per_seq = w.n_fac_per_seq.to(device)
        self.max_len = w.max_len
        self.T = w.total_tokens

    def kv(self, k_dom=None):
        return B.make_kv(self.k, self.v, self.offsets, self.max_len, self.T, k_dom)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def row_inputs(w, b, g):
    """float64 (q_group, keys, values) of row (b, g) of a Workload (exact upcasts of its bf16)."""
    G = w.spec.group
    o0, o1 = int(w.offsets[b]), int(w.offsets[b + 1])
    return (f64(w.q[b, g * G:(g + 1) * G]), f64(w.k[o0:o1, g]), f64(w.v[o0:o1, g]))


def check_device():
    st, detail = B.device_check()
    assert st == 0, f"device check fired: {detail}"


def score_bound(q_group, keys, idom):
    """sum over the scored dims of |q_c| |k_c| (the scale of the fp32 rounding of one score)."""
    return oracle.tip_scores(np.abs(q_group), np.abs(keys), idom)


U32 = 2.0 ** -24       # unit roundoff of fp32
WIDEN_CAP = 2e-2       # largest output-tolerance widening a band swap may claim (see output_tolerance)

# Session-wide record of how the tie band was used; printed at the end of the run (conftest).
BAND_STATS = {"rows": 0, "floor_binding": 0, "swapped": 0, "max_widening": 0.0}


def score_floor(q_group, keys, idom):
    """Absolute band floor: twice the worst fp32 rounding of any score of the row.

    The CUDA path sums the group's bf16 q heads in fp32 (G - 1 additions) and takes an fp32
    dot over the m = 2 n_dom scored dims; whatever the order, each score is then within
    gamma_{m+G} sum_h sum_c |q_hc| |k_c| of the exact one (gamma_k = k u / (1 - k u)).  Two
    tokens can swap places only when their exact scores are closer than twice that.
    """
    m = 2 * len(list(idom)) + q_group.shape[0]
    gamma = m * U32 / (1 - m * U32)
    bound = score_bound(q_group, keys, idom)
    return 2 * gamma * float(bound.max()) if bound.size else 0.0


def check_selection(gpu_sel, scores, n, floor):
    """The CUDA selection is a top-n of the oracle's scores up to the tie band; returns beta."""
    ok, msg = oracle.tie_band_check(gpu_sel, scores, n, BAND_REL, floor)
    assert ok, msg
    beta = oracle.tie_band(scores, n, BAND_REL, floor)
    BAND_STATS["rows"] += 1
    if n < len(scores) and n > 0 and floor > BAND_REL * abs(float(np.sort(scores)[::-1][n - 1])):
        BAND_STATS["floor_binding"] += 1
    return beta


def band_swap_bound(q_group, keys, values, scores, n, scale, beta):
    """Largest change of a head's output when band members are swapped (oracle values only).

    Tokens whose score lies within beta of the n-th score may be exchanged; attention over
    the kept core C moves by at most 2 max|v| * sum_band w / sum_C w.
    """
    s = np.asarray(scores)
    L = s.shape[0]
    if n >= L or n == 0:
        return 0.0
    s_n = np.sort(s)[::-1][n - 1]
    band = np.abs(s - s_n) <= beta
    core = s > s_n + beta
    worst = 0.0
    for h in range(q_group.shape[0]):
        z = scale * (keys @ q_group[h])
        z = z - z.max()
        w = np.exp(z)
        wc = w[core].sum()
        if wc <= 0:
            return np.inf
        worst = max(worst, 2 * np.abs(values).max() * w[band].sum() / wc)
    return worst


def output_tolerance(gpu_sel, ref_sel, q_attn, keys, values, scores, n, scale, beta):
    """OUT_ATOL, widened by the band-swap bound when the CUDA set differs inside the band.

    A swap of one band token moves an output by about |v_a - v_b| times its weight (about
    1/n of the core's), so the bound stays near 2 max|v| / n; WIDEN_CAP (2e-2, an order of
    magnitude above that for n in the hundreds) turns a bound that would hide a real
    selection drift (few core tokens, or an infinite bound) into a failure.
    """
    if np.array_equal(np.asarray(gpu_sel), np.asarray(ref_sel)):
        return OUT_ATOL
    widen = band_swap_bound(q_attn, keys, values, scores, n, scale, beta)
    BAND_STATS["swapped"] += 1
    BAND_STATS["max_widening"] = max(BAND_STATS["max_widening"], float(widen))
    assert widen <= WIDEN_CAP, f"band-swap widening {widen:.3g} above the cap {WIDEN_CAP}"
    return OUT_ATOL + widen


def compare_sparse_row(w, b, g, gpu_sel, gpu_out, stats=None):
    """Check one SPARSE row: selection within the tie band, output within 2e-3 of the oracle."""
    q_group, keys, values = row_inputs(w, b, g)
    idom = w.idom[g].tolist()
    n = int(min(int(w.n_fac_per_seq[b]), keys.shape[0]))
    s = oracle.tip_scores(q_group, keys, idom)
    beta = check_selection(gpu_sel, s, n, score_floor(q_group, keys, idom))
    ref_sel = oracle.select_top(s, n)
    ref_out = oracle.focused_attention(q_group, keys, values, ref_sel, w.scale)
    tol = output_tolerance(gpu_sel, ref_sel, q_group, keys, values, s, n, w.scale, beta)
    if stats is not None:
        stats["rows"] = stats.get("rows", 0) + 1
        stats["swapped"] = stats.get("swapped", 0) + (0 if tol == OUT_ATOL else 1)
    err = np.abs(gpu_out - ref_out).max() if ref_out.size else 0.0
    assert err <= tol, f"row ({b},{g}): max |out - oracle| = {err:.3g} > {tol:.3g}"
    return err


def compare_shared_row(w, b, g, gpu_sel, gpu_out_layers, topk):
    """One shared-index row: the index within the tie band of the indexer's full-dimension
    scores, every layer's output within 2e-3 of the oracle on its own index."""
    G = w.spec.group
    _, keys, values = row_inputs(w, b, g)
    qi = f64(w.q[b, g * G:(g + 1) * G])
    all_chunks = list(range(w.spec.head_dim // 2))
    s = oracle.tip_scores(qi, keys, all_chunks)
    n = min(topk, keys.shape[0])
    beta = check_selection(gpu_sel, s, n, score_floor(qi, keys, all_chunks))
    ref_sel = oracle.select_top(s, n)
    for l in range(gpu_out_layers.shape[0]):
        ql = f64(w.q_layers[l, b, g * G:(g + 1) * G])
        ref = oracle.focused_attention(ql, keys, values, ref_sel, w.scale)
        tol = output_tolerance(gpu_sel, ref_sel, ql, keys, values, s, n, w.scale, beta)
        err = np.abs(gpu_out_layers[l] - ref).max() if ref.size else 0.0
        assert err <= tol, f"row ({b},{g}) layer {l}: max err {err:.3g} > {tol:.3g}"


def compare_window_row(w, b, g, gpu_out, role, sink, window):
    q_group, keys, values = row_inputs(w, b, g)
    ref = oracle.decode_row(q_group, keys, values, role, w.scale, sink=sink, window=window)["out"]
    err = np.abs(gpu_out - ref).max() if ref.size else 0.0
    assert err <= OUT_ATOL, f"row ({b},{g}) role {role}: max err {err:.3g}"
    return err


def launches_of(fn) -> dict:
    """Kernels fn() launched through the library, by name (the library's launch counters)."""
    c0 = B.launch_counts()
    fn()
    torch.cuda.synchronize()
    c1 = B.launch_counts()
    return {k: c1[k] - c0[k] for k in c0 if c1[k] != c0[k]}


def three_kernel_form(launches: dict) -> bool:
    """scan + select + gather: the select is one cluster launch when every row's cluster fits
    one wave, else the row kernel's select-only launch for fewer rows than SMs, else the
    chunked select's four launches"""
    per_phase = ("select_hist_kernel", "select_chunk_kernel", "select_resolve_kernel", "select_write_kernel")
    others = lambda *ks: not any(k in launches for k in per_phase + ("select_cluster_kernel", "sparse_row_kernel")
                                 if k not in ks)
    on_chip = launches.get("select_cluster_kernel") == 1 and others("select_cluster_kernel")
    rows = launches.get("sparse_row_kernel") == 1 and others("sparse_row_kernel")
    chunked = all(launches.get(k) == 1 for k in per_phase) and others(*per_phase)
    return (launches.get("tip_score_kernel") == 1 and (on_chip or rows or chunked)
            and launches.get("flash_gather_kernel", 0) >= 1)


def run_sparse(d: Dev, pack=True):
    w = d.w
    step = SparseDecodeStep(d.k, d.v, d.offsets, d.max_len, d.T, w.spec.n_q_heads, w.roles.tolist(), w.scale,
                            idom=d.idom, n_fac=int(w.n_fac_per_seq.max()) if len(w.n_fac_per_seq) else 0,
                            n_fac_per_seq=d.n_fac_per_seq, n_fac_cap=max(1, int(w.n_fac_per_seq.max())),
                            sink=w.spec.sink, window=w.spec.window, pack_dominant=pack)
    out = step(d.q)
    torch.cuda.synchronize()
    check_device()
    return step, out


def run_shared(d: Dev, fused: bool = True):
    w = d.w
    step = SharedIndexStep(d.k, d.v, d.offsets, d.max_len, d.T, w.spec.n_layers, w.spec.n_q_heads,
                           w.spec.topk_shared, w.scale, fused=fused)
    out = step(d.q, d.q_layers)
    torch.cuda.synchronize()
    check_device()
    return step, out
