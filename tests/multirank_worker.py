"""One rank of the world_size-2 CPU test of the benchmark's multi-rank host logic
(run under torchrun with the gloo backend; each rank writes rank<r>.json into
the directory given as the first argument)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    ws, rank, _ = bench.dist_setup("gloo")
    import torch
    from kv_cache_vector_02_b200 import workloads as W
    # every rank gets the slowest rank's time
    t = bench.max_over_ranks(ws, 1.5 + rank, device="cpu")
    bench.barrier(ws)
    # each replica's batch is its own: a checksum of its first keys
    w = W.WORKLOADS["tiny"].with_(T=64, data_seed=bench.rank_data_seed(rank))
    k = W.gen_kv(w, 0)
    csum = float(k.float().abs().sum())
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(ws)]
    import torch.distributed as dist
    dist.all_gather(sums, torch.tensor([csum], dtype=torch.float64))
    rec = {"rank": rank, "ws": ws, "tmax": t, "sums": [float(s) for s in sums],
           "value": bench.whole_job_gbs(ws, 1e9, t)}
    with open(os.path.join(sys.argv[1], "rank%d.json" % rank), "w") as f:
        json.dump(rec, f)
    bench.barrier(ws)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
