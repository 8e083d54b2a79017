"""Parity of the CUDA path on caches that are not contiguous [T, Hkv, d] tensors.

The cache descriptor takes any 16-byte-aligned token and head strides.  Here the
same seeded inputs are stored two other ways and every operation must still match
the float64 oracle:
  * padded rows: each (token, head) row is d + 8 elements long, the last 8 unused
    (stride_head = d + 8, stride_tok = Hkv * (d + 8));
  * head-major: all tokens of head 0, then of head 1, ... (stride_tok = d,
    stride_head = T * d);
  * interleaved: the K row and the V row of a (token, head) side by side in one buffer
    [T, Hkv, 2, d] (v = k + d, stride_head = 2 * d, stride_tok = Hkv * 2 * d).
Both the fused one-launch form (few rows) and the three-kernel form (more rows
than one wave of clusters) are run, with the dominant columns packed and read in
place, at d = 64 and d = 128.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (Dev, check_device, compare_shared_row, compare_sparse_row, compare_window_row, f64,
                         launches_of, three_kernel_form)
from token_sparse_decode_b200 import binding as B
from token_sparse_decode_b200.step import SharedIndexStep, SparseDecodeStep
from workloads import ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, WorkloadSpec, make_workload

pytestmark = pytest.mark.gpu


def strided(t: torch.Tensor, layout: str) -> torch.Tensor:
    """A [T, Hkv, d] view of a copy of t stored in `layout`."""
    T, H, d = t.shape
    if layout == "padded":
        buf = torch.full((T, H, d + 8), float("nan"), dtype=t.dtype, device=t.device)
        buf[..., :d] = t
        view = buf[..., :d]
        assert view.stride() == (H * (d + 8), d + 8, 1)
        return view
    buf = t.permute(1, 0, 2).contiguous()  # [H, T, d]
    view = buf.permute(1, 0, 2)
    assert view.stride() == (d, T * d, 1)
    return view


def interleaved(k: torch.Tensor, v: torch.Tensor):
    """[T, Hkv, d] views of one [T, Hkv, 2, d] buffer holding copies of k and v."""
    T, H, d = k.shape
    buf = torch.stack([k, v], dim=2).contiguous()
    kv, vv = buf[:, :, 0, :], buf[:, :, 1, :]
    assert kv.stride() == vv.stride() == (H * 2 * d, 2 * d, 1)
    assert vv.data_ptr() - kv.data_ptr() == 2 * d
    return kv, vv


class StridedDev(Dev):
    def __init__(self, w, layout):
        super().__init__(w)
        if layout == "interleaved":
            self.k, self.v = interleaved(self.k, self.v)
        else:
            self.k = strided(self.k, layout)
            self.v = strided(self.v, layout)


def sparse_spec(d, batch, roles, seed):
    G = 4 if d == 128 else 2
    return WorkloadSpec(name="strided", batch=batch, n_q_heads=G * len(roles), n_kv_heads=len(roles), head_dim=d,
                        theta=5e5 if d == 128 else 1e4, len_range=(200, 5000), n_dom=16 if d == 128 else 5,
                        n_fac_div=8, roles=roles, sink=32, window=300, planted_frac=0.01, seed=seed)


@pytest.mark.parametrize("layout", ["padded", "head_major", "interleaved"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rows", ["few", "many"])
def test_role_split_step_on_strided_cache(layout, d, rows):
    roles = (ROLE_SPARSE, ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, ROLE_SPARSE, ROLE_SPARSE, ROLE_STREAM, ROLE_SPARSE)
    batch = 3 if rows == "few" else 40
    w = make_workload(sparse_spec(d, batch, roles, 700 + d + (0 if rows == "few" else 1)))
    dv = StridedDev(w, layout)
    for pack in (True, False):
        step = SparseDecodeStep(dv.k, dv.v, dv.offsets, dv.max_len, dv.T, w.spec.n_q_heads, w.roles.tolist(),
                                w.scale, idom=dv.idom, n_fac=int(w.n_fac_per_seq.max()),
                                n_fac_per_seq=dv.n_fac_per_seq, n_fac_cap=int(w.n_fac_per_seq.max()),
                                sink=w.spec.sink, window=w.spec.window, pack_dominant=pack)
        launched = launches_of(lambda: step(dv.q))
        if rows == "few":
            assert launched.get("sparse_row_kernel") == 1 and "tip_score_kernel" not in launched
        else:
            assert launched.get("tip_score_kernel") == 1 and launched.get("flash_gather_kernel", 0) >= 1
        check_device()
        out_h = f64(step.out)
        idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
        G = w.spec.group
        for b in range(0, batch, 1 if rows == "few" else 7):
            for g, role in enumerate(roles):
                o = out_h[b, g * G:(g + 1) * G]
                if role == ROLE_SPARSE:
                    compare_sparse_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], o)
                else:
                    compare_window_row(w, b, g, o, role, w.spec.sink, w.spec.window)


@pytest.mark.parametrize("layout", ["padded", "head_major", "interleaved"])
@pytest.mark.parametrize("batch", [2, 24])
def test_shared_index_step_on_strided_cache(layout, batch):
    sp = WorkloadSpec(name="strided_shared", batch=batch, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                      len_range=(500, 6000), n_layers=2, topk_shared=300, seed=720 + batch)
    w = make_workload(sp)
    dv = StridedDev(w, layout)
    step = SharedIndexStep(dv.k, dv.v, dv.offsets, dv.max_len, dv.T, sp.n_layers, sp.n_q_heads, sp.topk_shared,
                           w.scale)
    launched = launches_of(lambda: step(dv.q, dv.q_layers))
    if batch > 2:
        assert three_kernel_form(launched)
    check_device()
    out_h = f64(step.out)
    idx_h, cnt_h = step.idx.cpu().numpy(), step.count.cpu().numpy()
    G = sp.group
    for b in range(0, batch, 1 if batch == 2 else 5):
        for g in range(sp.n_kv_heads):
            compare_shared_row(w, b, g, idx_h[b, g, :cnt_h[b, g]], out_h[:, b, g * G:(g + 1) * G], sp.topk_shared)


def test_strided_and_contiguous_caches_give_the_same_bits():
    # the layout only moves where rows are read from: outputs and indices are identical
    roles = (ROLE_SPARSE,) * 4 + (ROLE_DENSE, ROLE_STREAM)
    w = make_workload(sparse_spec(128, 3, roles, 733))
    outs = []
    for dv in (Dev(w), StridedDev(w, "padded"), StridedDev(w, "head_major"), StridedDev(w, "interleaved")):
        step = SparseDecodeStep(dv.k, dv.v, dv.offsets, dv.max_len, dv.T, w.spec.n_q_heads, w.roles.tolist(),
                                w.scale, idom=dv.idom, n_fac=int(w.n_fac_per_seq.max()),
                                n_fac_per_seq=dv.n_fac_per_seq, n_fac_cap=int(w.n_fac_per_seq.max()),
                                sink=w.spec.sink, window=w.spec.window)
        step(dv.q)
        torch.cuda.synchronize()
        outs.append((step.out.clone(), step.idx.clone(), step.count.clone()))
    sparse = [g for g, r in enumerate(roles) if r == ROLE_SPARSE]  # idx / count rows of the other heads are not written
    for o, i, c in outs[1:]:
        assert torch.equal(o, outs[0][0])
        assert torch.equal(i[:, sparse], outs[0][1][:, sparse]) and torch.equal(c[:, sparse], outs[0][2][:, sparse])
    assert np.isfinite(f64(outs[0][0])).all()
    assert B.device_check()[0] == 0
