"""The no-allocation window-attention call against the workspace one.

Some callers cannot allocate device memory (their host owns every allocation,
or a cudaMalloc on their path is not allowed); for them the library offers
aoh_stream_decode_noalloc, which keeps its split-K scratch in a static device
array.  Here it must give the outputs of aoh_stream_decode on the same inputs,
on two calls in a row (the second call reuses the array the first one left
behind), and refuse a step whose scratch would not fit.  This file is collected
last so that a run stopping at the first failure has already run every other
test; it also passes alone in a fresh process.
"""


import numpy as np
import pytest
import torch

from token_sparse_decode_b200 import binding as B
from workloads import ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM, WorkloadSpec, make_workload

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3


def test_noalloc_matches_workspace_call_twice():
    roles = (ROLE_DENSE, ROLE_STREAM, ROLE_STREAM, ROLE_SPARSE, ROLE_DENSE, ROLE_STREAM, ROLE_STREAM, ROLE_STREAM)
    sp = WorkloadSpec(name="noalloc", batch=3, n_q_heads=32, n_kv_heads=8, head_dim=128, theta=5e5,
                      len_range=(300, 9000), roles=roles, sink=64, window=700, seed=601)
    w = make_workload(sp)
    dev = torch.device("cuda")
    k, v, q, offsets = w.k.to(dev), w.v.to(dev), w.q.to(dev), w.offsets.to(dev)
    kv = B.make_kv(k, v, offsets, w.max_len, w.total_tokens)
    ref = torch.full((3, 32, 128), 555.0, device=dev)
    ws = B.workspace(B.stream_decode_workspace_size(kv, 32, roles, sp.sink, sp.window), dev)
    B.stream_decode(q, kv, roles, sp.sink, sp.window, w.scale, ref, ws)
    torch.cuda.synchronize()
    ref_h = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full((3, 32, 128), 555.0, device=dev)
        B.stream_decode_noalloc(q, kv, roles, sp.sink, sp.window, w.scale, out)
        torch.cuda.synchronize()
        assert B.device_check()[0] == 0
        got = out.cpu().numpy()
        assert np.all(np.abs(got - ref_h) <= OUT_ATOL)
        # rows of SPARSE heads belong to the other call: untouched by both
        assert np.all(got[:, 12:16] == 555.0)


def test_noalloc_refuses_steps_beyond_its_scratch():
    # 512 one-token sequences x 8 dense KV heads = 4096 rows; their split-K partials need
    # about 17.06 MB, more than the 16 MiB array: refused on the host.  The buffers are
    # real and correctly sized, so that even a wrongly accepted call would stay in bounds.
    dev = torch.device("cuda")
    B_, Hkv, Hq, d = 512, 8, 32, 128
    k = torch.zeros((B_, Hkv, d), dtype=torch.bfloat16, device=dev)
    v = torch.zeros_like(k)
    q = torch.zeros((B_, Hq, d), dtype=torch.bfloat16, device=dev)
    offsets = torch.arange(B_ + 1, dtype=torch.int32, device=dev)
    kv = B.make_kv(k, v, offsets, 1, B_)
    roles = (ROLE_DENSE,) * Hkv
    need = B.stream_decode_workspace_size(kv, Hq, roles, 0, 0)
    assert need > (16 << 20)
    out = torch.full((B_, Hq, d), 7.0, device=dev)
    with pytest.raises(B.AohError) as e:
        B.stream_decode_noalloc(q, kv, roles, 0, 0, 0.088, out)
    assert e.value.status == 4  # AOH_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
