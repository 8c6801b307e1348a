"""The N > 1 host path of bench.py on CPU: two gloo ranks (one per process).

Each rank runs its own independent problem (weak scaling, no data-path
collective); the only collective is the max over ranks of the device time.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from frame_wise_linear_b200 import synth
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    assert bench.dist_env() == (world, rank, rank)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                  # this rank's device time
        job_ms = bench.max_over_ranks(ms, dist, "cpu")
        w = synth.WORKLOADS["tiny"]
        inp = synth.make_inputs(w, seed=rank)   # the bench seeds each rank's problem with its rank
        out[rank] = (job_ms, bench.job_value(w.units, world, job_ms), float(np.asarray(inp.K).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    world, port = 2, _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        for p in procs:
            if p.is_alive():
                p.kill()
                pytest.fail("a rank did not finish")
            assert p.exitcode == 0
        res = dict(out)
    from frame_wise_linear_b200 import synth
    w = synth.WORKLOADS["tiny"]
    for r in range(world):
        job_ms, value, _ = res[r]
        assert job_ms == 15.0                    # the slowest rank's time, on every rank
        assert value == pytest.approx(world * w.units / 15e-3)
    assert res[0][2] != res[1][2]                # independent problems per rank
    again = float(np.asarray(synth.make_inputs(w, seed=1).K).sum())
    assert again == res[1][2]                    # and each one reproducible


def test_backward_roofline_bytes_are_the_tensors():
    """The backward's algorithmic bytes: every input and gradient tensor once, summed from their shapes."""
    import bench
    from frame_wise_linear_b200 import synth
    for name in ("768p", "768p_h8", "mid"):
        w = synth.WORKLOADS[name]
        es = 2 if w.dtype == synth.DTYPE_BF16 else 4
        tok = (w.B, w.H, w.T, w.n)
        txt = (w.B, w.H, w.n_txt)
        shapes = [tok + (w.d_k,)] * 4 + [tok + (w.d_v,)] * 5 + [txt + (w.d_k,), txt + (w.d_v,)] * 2
        want = sum(int(np.prod(s)) for s in shapes) * es
        rf = bench.backward_roofline(w, {"hbm_gbs": 6549.1, "bf16_tflops": 1628.0})
        assert rf["bytes"] == want, name
    assert bench.backward_roofline(synth.WORKLOADS["768p"], {"hbm_gbs": 6549.1, "bf16_tflops": 1628.0})["bytes"] \
        == 3352690688


def test_forward_roofline_arithmetic():
    """The forward line's algorithmic bytes and path roofline at 768p (SURVEY's table: 1.862 GB, 284.3 us at
    the measured 6549.1 GB/s) and the e4m3 line's (Q, K, V, G and the text at one byte, O at two)."""
    import bench
    from frame_wise_linear_b200 import synth
    peaks = {"hbm_gbs": 6549.1, "bf16_tflops": 1628.3}
    w = synth.WORKLOADS["768p"]
    pr = bench.path_roofline(w, peaks)
    units, n, d, nt = w.B * w.H * w.T, w.n, w.d_k, w.n_txt
    want = 5 * units * n * d * 2 + 2 * w.B * w.H * nt * d * 2
    assert pr["bytes"] == want == 1862139904
    assert abs(pr["t_roof_s"] * 1e6 - 284.3) < 0.1
    assert bench.stage_work(w)["readout"]["bytes"] == 3 * units * n * d * 2      # Q, G read, O written
    w8 = synth.WORKLOADS["768p_fp8"]
    assert bench.path_roofline(w8, peaks)["bytes"] == 4 * units * n * d + units * n * d * 2 + 2 * w.B * w.H * nt * d


def test_softmax_work_counts_the_window():
    """The local softmax line's flops: 4 n keys d per query frame, keys = n x (window frames + anchors) + n_txt;
    at T = 45 the window and anchors allow 45 x 15 - 50 (the edge blocks have one neighbour) + 70 = 695 frame pairs."""
    import bench
    from frame_wise_linear_b200 import synth
    from oracle import softmax_oracle as so
    w = synth.WORKLOADS["768p"]
    pairs = sum(len(so.key_frames(t, w.T)) for t in range(w.T))
    assert pairs == 45 * 15 - 50 + 70
    want = 4 * w.B * w.H * w.n * w.d_k * (w.T * w.n_txt + pairs * w.n)
    assert bench.softmax_work(w) == want


def test_committed_dram_traffic_describes_the_current_forward_kernels():
    """profiles/dram_traffic.txt holds the ncu DRAM bytes of the 768p forward kernels for their current
    source files (the bench reports roofline.traffic only while the digests match)."""
    import bench
    from frame_wise_linear_b200 import synth
    w = synth.WORKLOADS["768p"]
    for stage in ("readout", "gram+factor", "scan"):
        assert bench.traffic_lookup(stage, w) is not None, stage
    algo = bench.stage_work(w)["readout"]["bytes"]
    assert 1.0 <= bench.traffic_lookup("readout", w) / algo < 1.2
