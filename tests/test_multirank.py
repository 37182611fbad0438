"""The multi-GPU data-parallel path, on two CPU ranks over gloo.

Requests are independent, so a multi-GPU run gives each rank its own shard
and puts no collective on the data path; the collectives only serve the
measurement (barrier, maximum of the ranks' times). Two ranks run as
separate processes (tests/mr_worker.py); each rank's result must equal a
single-process run of the same shard, the shards must differ, and the
measurement collectives must give the slowest rank's time and the
whole-job rate.
"""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

from quantized_linear_attention_sq_b200 import shards, synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _single_process(seed):
    import oracle

    w = synth.workload(0, seed=seed)
    c = w.cfg
    cal = w.calib()
    o_ = oracle.Oracle(c.batch, c.h_v, c.h_k, c.d, c.gate_kind, cal.unit_bits, cal.pivot, cal.col_scale,
                       cal.row_impact)
    pool = o_.new_pool()
    o_.quantize(pool, w.initial_state())
    outs = []
    for t in range(2):
        q, k, v, beta, g = w.step_inputs(t)
        o = np.zeros((c.batch, c.h_v, c.d), dtype=np.float32)
        o_.step(pool, q, k, v, beta, g, o=o)
        outs.append(o)
    return np.stack(outs), pool


def test_two_ranks_shard_requests_with_no_data_collective(tmp_path):
    world = 2
    port = _free_port()
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    procs = [subprocess.Popen([sys.executable, os.path.join(HERE, "mr_worker.py"), str(r), str(world), str(port),
                               str(tmp_path)], env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
             for r in range(world)]
    logs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            p.kill()
            out, _ = p.communicate()
        logs.append(out.decode(errors="replace"))
    for p, log in zip(procs, logs):
        assert p.returncode == 0, log[-2000:]
    res = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    # each rank owns a different shard ...
    assert int(res[0]["seed"]) != int(res[1]["seed"])
    assert not np.array_equal(res[0]["pool"], res[1]["pool"])
    # ... and its result is exactly that of a single process on the same shard
    for r in range(world):
        o_ref, pool_ref = _single_process(shards.rank_seed(11, r))
        assert np.abs(o_ref).max() > 0
        np.testing.assert_array_equal(res[r]["o"], o_ref)
        np.testing.assert_array_equal(res[r]["pool"], pool_ref)
    # measurement collectives: the slowest rank's time, the whole-job rate
    c = synth.CONFIGS[0]
    for r in range(world):
        assert float(res[r]["mx"]) == 10.0 * world
        assert float(res[r]["rate"]) == pytest.approx(world * c.batch * c.h_v * 2 / (10.0 * world / 1e3))


def test_single_process_helpers():
    assert shards.rank_seed(5, 0) == 5 and shards.rank_seed(5, 3) == 8
    assert shards.max_over_ranks(3.5) == 3.5
    assert shards.job_rate(100, 10, 250.0, 4) == pytest.approx(4 * 100 * 10 / 0.25)
