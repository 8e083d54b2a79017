"""Host logic of bench.py that decides what is measured: the algorithmic bytes of every
workload (closed forms of the step's reads), how many input copies keep each step cold, and
how bytes are attributed to the kernels of a fused or three-kernel call.  CPU only."""

from types import SimpleNamespace

import numpy as np
import torch

import bench
from workloads import preset
from workloads.synth import _draw_lengths, _draw_roles, _n_fac

L2 = 126 * 1024 * 1024


def lite(name):
    """The fields algorithmic_bytes reads, without generating the tensors."""
    spec = preset(name)
    lengths = _draw_lengths(spec)
    return SimpleNamespace(spec=spec, lengths=lengths, roles=torch.from_numpy(_draw_roles(spec)),
                           n_fac_per_seq=torch.from_numpy(_n_fac(spec, lengths)), max_len=int(lengths.max()))


def test_algorithmic_bytes_of_the_fixed_shape_workloads():
    # 8B-shaped layer: 32 rows x 32768 tokens x 16 chunks x 4 B, plus 32 x 2048 selected K+V rows of 512 B
    ab = bench.algorithmic_bytes(lite("llama8b_gqa4_L32k"))
    assert ab["tip"] == 32 * 32768 * 64 and ab["fac"] == 32 * 2048 * 512
    assert ab["total"] == 100663296
    # the same step with the scan reading K in place: the whole 256-byte K row of every token
    ab = bench.algorithmic_bytes(lite("llama8b_gqa4_L32k"), in_place=True)
    assert ab["tip"] == 32 * 32768 * 256 and ab["total"] == 32 * 32768 * 256 + 32 * 2048 * 512
    # AoH roles: 2 dense groups x 131072 tokens + 6 streaming groups x (128 + 4096) tokens, K+V rows of 512 B
    ab = bench.algorithmic_bytes(lite("aoh_roles_L128k"))
    assert ab["window"] == (2 * 131072 + 6 * 4224) * 512 == 147193856
    assert ab["total"] == ab["window"]
    # CLSA: full K rows of 2 x 8 x 131072 tokens (256 B) + one gather of 2 x 8 x 2048 K+V rows
    ab = bench.algorithmic_bytes(lite("clsa_shared_L128k"))
    assert ab["indexer"] == 2 * 8 * 131072 * 256 and ab["gather"] == 2 * 8 * 2048 * 512
    assert ab["total"] == 553648128
    # the select's score reads are reported per kernel, never counted as step traffic
    assert ab["select"] == 2 * 8 * 131072 * 4


def test_algorithmic_bytes_of_the_ragged_serving_batch():
    w = lite("fasa_serving_ragged_b64")
    L = w.lengths.astype(np.int64)
    assert len(L) == 64 and L.min() >= 4096 and L.max() <= 65536
    n = -(-L // 8)  # ceil(L / 8) selected tokens per sequence
    ab = bench.algorithmic_bytes(w)
    assert ab["tip"] == int(L.sum()) * 4 * 64
    assert ab["fac"] == int(n.sum()) * 4 * 512
    assert ab["total"] == ab["tip"] + ab["fac"]


def test_cold_copies():
    assert bench.cold_copies(100663296, L2) == 4   # 3 x 100.7 MB >= 2 x 126 MB > 2 x 100.7 MB
    assert bench.cold_copies(147193856, L2) == 3
    assert bench.cold_copies(553648128, L2) == 2
    assert bench.cold_copies(2 * L2, L2) == 2      # exactly two L2 sizes between reuses
    assert bench.cold_copies(80_000, L2) == 0      # too small: flush instead
    # the other copies move at least 2 x L2 between two uses of a copy, and R is the smallest such
    for b in (40_000_000, 63_000_000, 64_000_000, 300_000_000):
        r = bench.cold_copies(b, L2)
        assert r >= 2
        assert (r - 1) * b >= 2 * L2
        assert r == 2 or (r - 2) * b < 2 * L2


def test_kernel_bytes_follow_the_path_taken():
    w = lite("llama8b_gqa4_L32k")
    ab = bench.algorithmic_bytes(w)
    fused = ["sparse_row_kernel"]
    three = ["tip_score_kernel", "select_chunk_kernel", "select_write_kernel", "flash_gather_kernel"]
    assert bench.kernel_bytes(w, ab, "decode_step", "sparse_row_kernel", fused) == ab["tip"] + ab["fac"]
    assert bench.kernel_bytes(w, ab, "decode_step", "tip_score_kernel", three) == ab["tip"]
    assert bench.kernel_bytes(w, ab, "decode_step", "select_chunk_kernel", three) == ab["select"]
    assert bench.kernel_bytes(w, ab, "decode_step", "flash_gather_kernel", three, 3) == ab["fac"]
    # a second gather in the same call attends the window heads; without a scan every gather does
    t = lite("tiny_mixed_d64_L512")
    abt = bench.algorithmic_bytes(t)
    assert bench.kernel_bytes(t, abt, "decode_step", "sparse_row_kernel", fused) == abt["tip"] + abt["fac"] + abt["window"]
    assert bench.kernel_bytes(t, abt, "decode_step", "flash_gather_kernel", three + ["flash_gather_kernel"], 4) == abt["window"]
    a = lite("aoh_roles_L128k")
    aba = bench.algorithmic_bytes(a)
    assert bench.kernel_bytes(a, aba, "decode_step", "flash_gather_kernel", ["flash_gather_kernel"], 0) == aba["window"]
    c = lite("clsa_shared_L128k")
    abc = bench.algorithmic_bytes(c)
    assert bench.kernel_bytes(c, abc, "shared_index_step", "sparse_row_kernel", fused) == abc["total"]
    assert bench.kernel_bytes(c, abc, "shared_index_step", "select_write_kernel", three) == abc["select"]
    assert bench.kernel_bytes(c, abc, "shared_index_step", "flash_gather_kernel", three) == abc["gather"]


def test_both_arms_report_the_same_config():
    # the reference arm and ours describe the workload with the same keys and values
    w = lite("clsa_shared_L128k")
    cfg = bench.workload_config(w, 1)
    assert cfg["workload"] == "clsa_shared_L128k" and cfg["algorithmic_bytes_per_step"] == 553648128
    assert cfg["tokens_per_step_per_gpu"] == 2 * 131072 and cfg["n_layers"] == 8
    assert cfg["parallelism"] == "independent sequences per rank x1"


def test_gpus_flag_relaunches_under_torchrun():
    cmd = bench.torchrun_command(4, 29555, ["--gpus", "4", "--steps", "7"])
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd and "--master-port=29555" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "4", "--steps", "7"] and cmd[-5].endswith("bench.py")


def test_oracle_pool_sizing_and_core_report():
    cores = bench.host_cores()
    assert cores["affinity_cores"] >= 1 and cores["host_cpu_count"] >= cores["affinity_cores"]
    assert 1 <= bench.pool_size(None) <= min(bench.MAX_POOL, cores["affinity_cores"])
    assert bench.repeats_for(5.0) == 1          # a long row runs once per batch
    assert bench.repeats_for(0.01, 1.0) == 100  # short rows repeat to about a second of work
    assert bench.repeats_for(0.0) >= 1


def test_row_tasks_carry_compact_copies():
    from workloads import make_workload

    w = make_workload(preset("tiny_mixed_d64_L512"))
    task, n = bench.row_task(w, 0, 3)
    assert n == 512 and task[0] == "row" and task[4] == int(w.roles[3])
    keys = task[2]
    assert keys.is_contiguous() and keys.shape == (512, 64) and keys.untyped_storage().nbytes() == 512 * 64 * 2
    assert bench.oracle_row(task) > 0
