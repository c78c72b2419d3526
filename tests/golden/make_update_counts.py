"""Write update_counts.txt: the exact number of positive-length ray-voxel
segments of each seeded workload, counted by the FP64 oracle (and by nothing
else).  Runs the oracle over view ranges in parallel processes.

    python tests/golden/make_update_counts.py [workload ...]
"""
import json
import multiprocessing as mp
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)


def _count(args):
    import oracle
    from ray_forward_back_b200 import workloads as W
    index, v0, v1 = args
    return index, oracle.count_updates(W.workload(index).geom, (v0, v1))


def main(indices):
    import oracle
    from ray_forward_back_b200 import workloads as W
    oracle.build()
    tasks = []
    for i in indices:
        nv = W.workload(i).geom.n_views
        edges = np.linspace(0, nv, 33).round().astype(int)
        tasks += [(i, int(a), int(b)) for a, b in zip(edges[:-1], edges[1:]) if b > a]
    with mp.get_context("spawn").Pool(os.cpu_count()) as pool:
        parts = pool.map(_count, tasks)
    totals = {i: 0 for i in indices}
    for i, n in parts:
        totals[i] += n
    path = os.path.join(HERE, "update_counts.txt")
    with open(path, "w") as f:
        f.write("# Exact positive-length ray-voxel segment counts of the seeded workloads,\n")
        f.write("# counted by the FP64 oracle (tests/golden/make_update_counts.py).\n")
        f.write("# columns: workload index, count\n")
        for i in indices:
            f.write(f"{i} {totals[i]}\n")
    print(json.dumps(totals))


if __name__ == "__main__":
    main([int(a) for a in sys.argv[1:]] or [0, 1, 2, 3])
