"""The C ABI on the CPU: the library loads, exports every declared symbol, its
struct layout matches the header, and host-side validation rejects bad calls
before anything reaches a GPU (no compute call is made here)."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch  # noqa: F401  (loads torch's CUDA runtime first, as in real use)

from token_sparse_decode_b200 import binding as B
from token_sparse_decode_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "aoh.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(aoh_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTS)


def test_version_and_status_strings(lib):
    assert lib.aoh_version() == 2
    assert lib.aoh_status_string(0) == b"ok"
    assert lib.aoh_status_string(4).startswith(b"workspace")
    assert lib.aoh_status_string(99) == b"unknown status"


def test_launch_counters_are_host_side(lib):
    # the kernel-kind enum of the header and the binding's names agree, and the counters
    # read without a device; host validation failures launch nothing
    text = open(HEADER).read()
    kinds = re.findall(r"AOH_KERNEL_([A-Z_]+) = (\d+)", text)
    named = {k.lower(): int(v) for k, v in kinds if k != "KINDS"}
    assert [f"{k}_kernel" for k, _ in sorted(named.items(), key=lambda kv: kv[1])] == list(B.KERNELS)
    before = B.launch_counts()
    assert set(before) == set(B.KERNELS) and all(v >= 0 for v in before.values())
    assert lib.aoh_launch_counts(None, 0) == len(B.KERNELS)
    kv = B.KVCache()
    kv.batch, kv.n_kv_heads, kv.head_dim = 1, 1, 96  # unsupported head_dim: refused on the host
    assert lib.aoh_tip_score(None, 1, ctypes.byref(kv), None, 1, None, None) == 2
    assert B.launch_counts() == before


def test_struct_layout_matches_header():
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "aoh.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(aoh_kv_cache), offsetof(aoh_kv_cache, batch),
             offsetof(aoh_kv_cache, total_tokens), offsetof(aoh_kv_cache, stride_head),
             offsetof(aoh_kv_cache, k_dom), offsetof(aoh_kv_cache, k_dom_cols),
             offsetof(aoh_kv_cache, lengths), offsetof(aoh_kv_cache, head_slot),
             offsetof(aoh_kv_cache, ring_sink), offsetof(aoh_kv_cache, ring_window));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()]
    K = B.KVCache
    assert vals == [ctypes.sizeof(K), K.batch.offset, K.total_tokens.offset, K.stride_head.offset,
                    K.k_dom.offset, K.k_dom_cols.offset, K.lengths.offset, K.head_slot.offset,
                    K.ring_sink.offset, K.ring_window.offset]


def fake_kv(**kw):
    kv = B.KVCache()
    kv.k, kv.v, kv.offsets = 0x10000, 0x20000, 0x30000
    kv.batch, kv.n_kv_heads, kv.head_dim, kv.max_len = 2, 8, 128, 1000
    kv.total_tokens, kv.stride_tok, kv.stride_head = 2000, 8 * 128, 128
    for a, b in kw.items():
        setattr(kv, a, b)
    return kv


def call_sparse(lib, kv, **kw):
    a = dict(q=0x40000, hq=32, idom=0x50000, n_dom=16, n_fac=64, nfps=None, cap=64, roles=None, scale=0.088,
             out=0x60000, idx=None, cnt=None, ws=0x70000, ws_bytes=1 << 40)
    a.update(kw)
    return lib.aoh_sparse_decode(a["q"], a["hq"], ctypes.byref(kv), a["idom"], a["n_dom"], a["n_fac"], a["nfps"],
                                 a["cap"], a["roles"], a["scale"], a["out"], a["idx"], a["cnt"], a["ws"],
                                 a["ws_bytes"], None)


def test_host_validation_rejects_before_launch(lib):
    INVALID, UNSUP, ALIGN, WS = 1, 2, 3, 4
    assert lib.aoh_tip_score(0x40000, 32, None, 0x50000, 16, 0x60000, None) == INVALID
    assert call_sparse(lib, fake_kv(head_dim=96)) == UNSUP
    assert call_sparse(lib, fake_kv(k=0x10008)) == ALIGN            # K not 16-byte aligned
    assert call_sparse(lib, fake_kv(stride_tok=8 * 128 + 4)) == ALIGN
    assert call_sparse(lib, fake_kv(), hq=30) == INVALID            # Hq % Hkv != 0
    assert call_sparse(lib, fake_kv(), n_dom=65) == INVALID         # n_dom > d/2
    assert call_sparse(lib, fake_kv(), n_dom=0) == INVALID
    assert call_sparse(lib, fake_kv(), n_fac=65, cap=64) == INVALID  # N_fac above capacity
    assert call_sparse(lib, fake_kv(), ws=None) == WS
    assert call_sparse(lib, fake_kv(), ws_bytes=100) == WS
    assert call_sparse(lib, fake_kv(), ws=0x70010) == WS            # not 256-byte aligned
    assert call_sparse(lib, fake_kv(), q=None) == INVALID
    assert call_sparse(lib, fake_kv(), q=0x40004) == ALIGN
    assert call_sparse(lib, fake_kv(), scale=float("nan")) == INVALID
    assert call_sparse(lib, fake_kv(n_kv_heads=0)) == INVALID
    assert call_sparse(lib, fake_kv(total_tokens=1 << 31)) == INVALID
    bad_roles = (ctypes.c_uint8 * 8)(0, 1, 2, 3, 0, 0, 0, 0)
    assert call_sparse(lib, fake_kv(), roles=ctypes.cast(bad_roles, ctypes.c_void_p)) == INVALID
    assert call_sparse(lib, fake_kv(batch=0)) == 0                  # empty batch is a no-op
    roles = (ctypes.c_uint8 * 8)(*([2] * 8))
    r = ctypes.cast(roles, ctypes.c_void_p)
    assert lib.aoh_stream_decode(0x40000, 32, ctypes.byref(fake_kv()), None, 4, 60, 0.1, 0x60000, 0x70000,
                                 1 << 40, None) == INVALID          # roles required
    assert lib.aoh_stream_decode(0x40000, 32, ctypes.byref(fake_kv()), r, -1, 60, 0.1, 0x60000, 0x70000,
                                 1 << 40, None) == INVALID
    # shared index: more than 32 query rows per KV head
    assert lib.aoh_shared_index_decode(0x40000, 9, 32, ctypes.byref(fake_kv()), 0x50000, 0x58000, 64, 0.1,
                                       0x60000, 0x70000, 1 << 40, None) == UNSUP
    assert lib.aoh_topk_select(0x40000, ctypes.byref(fake_kv()), 10, None, 0, 0x50000, 0x58000, 0x70000, 1 << 40,
                               None) == INVALID
    assert lib.aoh_topk_select(0x40000, ctypes.byref(fake_kv()), 10, None, 64, 0x50000, 0x58000, None, 0,
                               None) == WS
    assert lib.aoh_topk_select_workspace_size(ctypes.byref(fake_kv())) >= 8 * 2000 * 8  # the candidate lists
    assert lib.aoh_pack_dominant(ctypes.byref(fake_kv()), 0x50000, 16, 0x60000, 36, None) == INVALID


def test_workspace_sizes_are_host_computations(lib):
    kv = fake_kv()
    s = lib.aoh_sparse_decode_workspace_size(ctypes.byref(kv), 32, 2048)
    # at least the fp32 score row of every head plus the index
    assert s >= 4 * 8 * 2000 + 4 * 2 * 8 * 2048
    assert s % 256 == 0
    roles = (ctypes.c_uint8 * 8)(*([1, 2] * 4))
    assert lib.aoh_stream_decode_workspace_size(ctypes.byref(kv), 32, ctypes.cast(roles, ctypes.c_void_p), 4, 60) > 0
    assert lib.aoh_shared_index_decode_workspace_size(ctypes.byref(kv), 8, 32, 2048) > 0
    assert lib.aoh_shared_index_decode_workspace_size(ctypes.byref(kv), 9, 32, 2048) == 0
    assert lib.aoh_sparse_decode_workspace_size(ctypes.byref(fake_kv(head_dim=96)), 32, 64) == 0


def test_ring_and_append_rules_are_checked_on_the_host(lib):
    INVALID = 1
    ring = fake_kv(ring_sink=16, ring_window=64)
    roles = (ctypes.c_uint8 * 8)(*([2] * 8))            # every head STREAM
    r = ctypes.cast(roles, ctypes.c_void_p)
    # a ring serves streaming heads within its sink and window, and nothing else
    assert call_sparse(lib, ring) == INVALID
    assert lib.aoh_tip_score(0x40000, 32, ctypes.byref(ring), 0x50000, 16, 0x60000, None) == INVALID
    assert lib.aoh_pack_dominant(ctypes.byref(ring), 0x50000, 16, 0x60000, 32, None) == INVALID
    assert lib.aoh_stream_decode(0x40000, 32, ctypes.byref(ring), r, 17, 64, 0.1, 0x60000, 0x70000,
                                 1 << 40, None) == INVALID  # sink beyond the ring's
    assert lib.aoh_stream_decode(0x40000, 32, ctypes.byref(ring), r, 16, 65, 0.1, 0x60000, 0x70000,
                                 1 << 40, None) == INVALID  # window beyond the ring's
    dense = (ctypes.c_uint8 * 8)(1, 2, 2, 2, 2, 2, 2, 2)
    assert lib.aoh_stream_decode(0x40000, 32, ctypes.byref(ring), ctypes.cast(dense, ctypes.c_void_p), 16, 64, 0.1,
                                 0x60000, 0x70000, 1 << 40, None) == INVALID  # a DENSE head stored in a ring
    # ... unless the ring does not store that head
    slots = (ctypes.c_uint8 * 8)(255, 0, 1, 2, 3, 4, 5, 6)
    ring2 = fake_kv(ring_sink=16, ring_window=64, head_slot=ctypes.cast(slots, ctypes.c_void_p).value)
    assert lib.aoh_stream_decode_workspace_size(ctypes.byref(ring2), 32, ctypes.cast(dense, ctypes.c_void_p),
                                                16, 64) > 0
    # append: a linear cache and a ring, every head kept somewhere, lengths required
    lin = fake_kv()
    app = lib.aoh_kv_append
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, None, None, None, 0, 0x60000, 0x68000, None) == INVALID
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, ctypes.byref(ring), None, None, 0, 0x60000, 0x68000,
               None) == INVALID                       # a ring given as the linear cache
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, None, ctypes.byref(lin), None, 0, 0x60000, 0x68000,
               None) == INVALID                       # a linear cache given as the ring
    only_two = (ctypes.c_uint8 * 8)(0, 1, 255, 255, 255, 255, 255, 255)
    part = fake_kv(head_slot=ctypes.cast(only_two, ctypes.c_void_p).value)
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, ctypes.byref(part), None, None, 0, 0x60000, 0x68000,
               None) == INVALID                       # heads 2..7 kept nowhere
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, ctypes.byref(lin), None, None, 0, None, 0x68000,
               None) == INVALID                       # no lengths
    assert app(0x40000, 32, 0x50000, 0x58000, -1.0, ctypes.byref(lin), None, None, 0, 0x60000, 0x68000,
               None) == INVALID                       # theta <= 0
    assert app(0x40000, 32, 0x50000, 0x58000, 5e5, ctypes.byref(lin), None, None, 0, 0x60000, None,
               None) == INVALID                       # q without q_out
    packed = fake_kv(k_dom=0x80000, k_dom_cols=32)
    assert app(None, 0, 0x50000, 0x58000, 5e5, ctypes.byref(packed), None, None, 0, 0x60000, None,
               None) == INVALID                       # k_dom without I_dom
    assert app(None, 0, 0x50000, 0x58000, 5e5, ctypes.byref(fake_kv(batch=0)), None, None, 0, None, None,
               None) == 0                             # empty batch: nothing to do


def test_head_classifier_arguments_are_checked_on_the_host(lib):
    INVALID, UNSUP, ALIGN, WS = 1, 2, 3, 4
    cls = lib.aoh_head_classify
    ok = dict(wq=0x10000, wk=0x20000, dm=4096, hq=32, hkv=8, d=128, nr=4, eh=0x30000, eg=0x38000, r=0x40000,
              ws=0x50000, wsb=1 << 40)

    def call(**kw):
        a = dict(ok, **kw)
        return cls(a["wq"], a["wk"], a["dm"], a["hq"], a["hkv"], a["d"], a["nr"], a["eh"], a["eg"], a["r"], a["ws"],
                   a["wsb"], None)

    assert call(d=96) == UNSUP
    assert call(hq=30) == INVALID            # q heads not a multiple of the KV heads
    assert call(dm=4000) == INVALID          # d_model not a multiple of 64
    assert call(dm=64) == INVALID            # d_model below head_dim
    assert call(nr=9) == INVALID and call(nr=-1) == INVALID
    assert call(wq=0x10008) == ALIGN
    assert call(eh=None) == INVALID
    assert call(ws=None) == WS and call(wsb=1000) == WS
    size = lib.aoh_head_classify_workspace_size
    need = size(4096, 32, 8, 128)
    # fp64 partials of 8 splits of 512 columns, fp64 Gram matrices of 40 heads, fp64 scratch of 32
    assert need == 40 * 8 * 128 * 128 * 8 + 40 * 128 * 128 * 8 + 32 * 128 * 128 * 8
    assert size(4096, 30, 8, 128) == 0 and size(192, 4, 2, 64) > 0
