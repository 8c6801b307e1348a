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
