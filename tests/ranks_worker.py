"""One rank of the multi-rank host-logic test (run as a subprocess with RANK,
WORLD_SIZE, LOCAL_RANK, MASTER_ADDR and MASTER_PORT set): gloo process group,
the bench's max-over-ranks timing and whole-job throughput; prints one JSON
line."""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

r = bench.Ranks("gloo", timeout_s=60)
own_ms = 10.0 + r.rank  # each rank's own device time
slowest = r.max(own_ms)
r.barrier()
value = bench.job_throughput(r.world, 100, slowest)
r.close()
print(json.dumps({"rank": r.rank, "world": r.world, "max_ms": slowest, "value": value}))
