"""Multi-process (world size 2, gloo, CPU) checks of the data-parallel host
logic: row shards cover every token exactly once, per-rank results computed
on the shards reassemble to the single-process result, and the reported time
is the max over ranks.  The layer itself needs a B200; here each rank runs
the CPU oracle on its shard, which is exactly the computation the GPU rank
performs on its rows (no data-path collective exists to test)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        from quantized_gemm_token_b200.dist import max_over_ranks, shard_rows

        d = synth.tiny(0)
        M = d["x"].shape[0] + 3                    # ragged: 67 rows over 2 ranks
        x = np.concatenate([d["x"], d["x"][:3]])
        start, stop = shard_rows(M, world, rank)
        wq, sc = oracle.quantize_rows_f32(d["w"])
        out, _, _ = oracle.dynamic_linear_bf16(x[start:stop], wq, sc, d["bias"])
        # gather only to verify (the layer itself has no collective)
        parts = [None] * world
        dist.all_gather_object(parts, (start, stop, out))
        t = max_over_ranks(10.0 + rank)
        if rank == 0:
            full, _, _ = oracle.dynamic_linear_bf16(x, wq, sc, d["bias"])
            rows = sorted((p[0], p[1]) for p in parts)
            ok_cover = rows[0][0] == 0 and rows[-1][1] == M and all(
                rows[i][1] == rows[i + 1][0] for i in range(len(rows) - 1))
            stitched = np.concatenate([p[2] for p in sorted(parts, key=lambda p: p[0])])
            result_q.put((ok_cover, bool(np.array_equal(stitched, full)), t))
    finally:
        dist.destroy_process_group()


def test_row_shards_partition_and_reassemble_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    ok_cover, ok_equal, t = q.get(timeout=5)
    assert ok_cover and ok_equal
    assert t == 11.0                               # max over ranks


@pytest.mark.parametrize("M,world", [(0, 2), (1, 2), (7, 3), (2048, 8), (65792, 8)])
def test_shard_rows_balanced(M, world):
    from quantized_gemm_token_b200.dist import shard_rows
    spans = [shard_rows(M, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == M
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
    assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
