"""One rank of the host-side multi-rank tests (run as a subprocess with
RANK / WORLD_SIZE / MASTER_* set).  Uses bench.py's own distributed helpers
on the gloo backend; prints one JSON line with what this rank saw."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    mode = sys.argv[1]
    rank, world, _ = bench.dist_init(world_size := int(os.environ["WORLD_SIZE"]),
                                     timeout_s=float(os.environ.get("PG_TIMEOUT_S", "20")))
    import torch.distributed as dist
    out = {"rank": rank, "world": world, "backend": dist.get_backend()}
    if mode == "max":
        # Per-rank "times" 1.5, 2.5, ...: every rank must see the slowest.
        bench.barrier(world)
        out["max"] = bench.max_over_ranks(1.5 + rank, world)
        out["value"] = bench.replica_value(4.0e6, world, out["max"])
        bench.barrier(world)
    elif mode == "dead_peer":
        # Rank 1 leaves between steps (no collective in flight); rank 0 must
        # learn of it from its next collective as an error, not a hang.
        if rank == 1:
            print(json.dumps(out), flush=True)
            os._exit(0)
        try:
            bench.barrier(world)
            out["error"] = None
        except Exception as e:  # the process group reports the missing peer
            out["error"] = type(e).__name__
        print(json.dumps(out), flush=True)
        os._exit(0)
    print(json.dumps(out), flush=True)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
