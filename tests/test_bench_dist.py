"""Multi-rank plumbing of bench.py on CPU: world_size 2 over gloo.

The decode path has no exchange step (every rank runs its own replica), so the
only cross-rank operations are the timing and byte-count reductions: the
job's time is the max over ranks and its bytes the sum.  The reference arm
runs on rank 0 alone.
"""

from __future__ import annotations

import datetime
import io
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
        import torch
        import torch.distributed as dist

        import bench

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        cpu = torch.device("cpu")
        # each rank "measured" a different time and processed its own bytes
        t_max = bench.reduce_max(10.0 + rank, True, cpu)
        b_sum = bench.reduce_sum(1000.0 * (rank + 1), True, cpu)
        # without torch.distributed both are the identity
        ident = (bench.reduce_max(3.5, False), bench.reduce_sum(3.5, False))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, t_max, b_sum, ident))
    except Exception as e:  # report, never hang the parent
        q.put((rank, "error", repr(e), None))


@pytest.mark.timeout(180)
def test_reductions_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, t_max, b_sum, ident in results:
        assert t_max != "error", b_sum
        assert t_max == 11.0          # the slowest rank's time
        assert b_sum == 3000.0        # all ranks' bytes
        assert ident == (3.5, 3.5)


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    out = io.StringIO()
    with redirect_stdout(out):
        bench.run_reference_arm(bench.parse_args(["--impl", "reference", "--steps", "3", "--warmup", "3"]))
    assert out.getvalue() == ""


def test_warmup_floor():
    sys.path.insert(0, ROOT)
    import bench

    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    assert bench.parse_args([]).warmup >= 3


def test_profiled_traffic_only_for_matching_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from profiles/traffic.json only while the CUDA sources match its hash."""
    import json
    sys.path.insert(0, ROOT)
    import bench

    p = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(p))
    assert bench.profiled_traffic("w") is None                  # no file
    p.write_text(json.dumps({"w": {"bytes_per_step": 12345, "csrc_sha256": bench.csrc_sha256()}}))
    assert bench.profiled_traffic("w") == 12345
    assert bench.profiled_traffic("other") is None              # no record for that workload
    p.write_text(json.dumps({"w": {"bytes_per_step": 12345, "csrc_sha256": "0" * 64}}))
    assert bench.profiled_traffic("w") is None                  # kernels changed since the capture


def test_fused_layer_is_the_layer_with_rows_concatenated():
    """The fused Q4_K layer stacks q, k, v and gate, up row-wise: the same weights and bytes in 4 calls, not 7."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench

    plain = bench.step_calls("q4_k_7b_layer_decode")
    fused = bench.step_calls("q4_k_7b_layer_decode_fused")
    assert len(plain) == 7 and len(fused) == 4
    wbytes = lambda calls: sum(N * bench.inputs.row_bytes(f, K) for f, a, M, N, K, s in calls)
    assert wbytes(plain) == wbytes(fused)
    # weights generated at reduced K so the check stays fast: stacking commutes with generation
    f, a, M, N, K, seed = fused[0]
    K = 256
    stacked = bench.call_weights(f, N, K, seed)
    parts = [bench.call_weights(f, N // 3, K, s) for s in seed]
    assert np.array_equal(stacked, np.concatenate(parts, axis=0))
    assert stacked.shape == (N, bench.inputs.row_bytes(f, K))


class _Graph:
    def __init__(self, tag, log):
        self.tag, self.log = tag, log

    def replay(self):
        self.log.append(self.tag)


@pytest.mark.parametrize("R,W,K", [(7, 3, 10), (7, 10, 25), (30, 3, 12), (5, 5, 5), (3, 4, 7), (4, 0, 9)])
def test_replay_steps_times_exactly_k_steps(R, W, K):
    """Whole rotations replay one R-step graph, the rest one-step graphs; the warm-up ends on
    copy R-1, and the timed steps read copies 0, 1, 2, ... in order."""
    sys.path.insert(0, ROOT)
    import bench

    log = []
    singles = [_Graph(r, log) for r in range(R)]
    full = _Graph("full", log)
    bench.replay_steps(singles, full, W, first=-W)
    warm = list(log)
    log.clear()
    bench.replay_steps(singles, full, K)
    expand = lambda seq: [c for t in seq for c in (range(R) if t == "full" else [t])]
    assert expand(warm) == [(R - W + i) % R for i in range(W)]
    assert expand(log) == [i % R for i in range(K)]


def test_int8_workload_codes():
    sys.path.insert(0, ROOT)
    import bench
    import block_quantized_matmul_lwq_b200 as lwq

    calls = bench.step_calls("q4_0_gemv_11008x4096_act_i8")
    assert [c[2] for c in calls] == [1, 4, 8]
    f, a, M, N, K, s = calls[0]
    assert bench.base_act(a) == "f32"
    assert bench.call_fmt(lwq, f, a) == lwq.fmt_code("q4_0", "f32") | lwq.LWQ_FLAG_ACT_I8
    assert bench.call_fmt(lwq, f, "f32") == lwq.fmt_code("q4_0", "f32")
    # the same bytes as the fp32 step: packed weights, fp32 x, fp32 y
    assert bench.call_bytes(f, a, M, N, K) == bench.call_bytes(f, "f32", M, N, K)
