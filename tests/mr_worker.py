"""One rank of the two-rank CPU test of the data-parallel plumbing (gloo).

    python tests/mr_worker.py RANK WORLD PORT OUT_DIR

Each rank builds its own shard of a small seeded workload (the plumbing
workload: batch 1, 4 heads, d = 64), steps it through the CPU oracle with
no collective on the data path, then exercises the measurement
collectives (max over ranks, whole-job rate) and writes what it saw to
OUT_DIR/rank<RANK>.npz.
"""
import datetime
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main():
    rank, world, port, out_dir = int(sys.argv[1]), int(sys.argv[2]), int(sys.argv[3]), sys.argv[4]
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from quantized_linear_attention_sq_b200 import shards, synth

        seed = shards.rank_seed(11, rank)
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
        dist.barrier()
        mx = shards.max_over_ranks(float(10 * (rank + 1)), dist)
        rate = shards.job_rate(c.batch * c.h_v, 2, mx, world)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), seed=seed, o=np.stack(outs), pool=pool, mx=mx,
                 rate=rate)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
