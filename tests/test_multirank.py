"""Host logic of the multi-GPU benchmark path, on CPU with gloo, world sizes 2 and 4.

Every rank runs its own independent batch (weak scaling, no data-path
collective); the only cross-rank steps are the barrier and the max over ranks
of the timed region.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    import bench
    from gated_delta_rule_109_b200 import inputs as I
    try:
        r, lr, ws = bench.init_distributed(backend="gloo", timeout_s=60)
        w = bench.rank_workload(I.PREFILL_H32_T64K, r)
        bench.barrier()
        mx = bench.max_over_ranks(10.0 + 5.0 * r)
        # the reference arm: ranks other than 0 exit at once without work
        class A:
            pass
        a = A()
        a.steps, a.warmup, a.ref_tokens_per_step = 1, 3, 16
        rc_ref = bench.run_reference(a) if r != 0 else 0
        q.put((r, ws, w.seed, w.T, mx, rc_ref))
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 4])
def test_weak_scaling_host_logic(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=200) for _ in procs]
    for p in procs:
        p.join(timeout=30)
    assert all(len(x) == 6 for x in res), res
    res.sort()
    assert [x[0] for x in res] == list(range(world))
    assert all(x[1] == world for x in res)
    assert len({x[2] for x in res}) == world                 # independent batches ...
    assert all(x[3] == 65536 for x in res)                   # ... of the same size
    assert all(x[4] == 10.0 + 5.0 * (world - 1) for x in res)   # max over ranks, seen by every rank
    assert all(x[5] == 0 for x in res[1:])                   # reference arm: ranks > 0 do no work


def test_single_process_helpers_are_identities():
    import bench
    from gated_delta_rule_109_b200 import inputs as I
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_workload(I.PREFILL_H32_T64K, 0).seed == I.PREFILL_H32_T64K.seed
    assert bench.prefill_bytes_per_token_head(128, 128, 2) == 1796
    assert bench.prefill_flops_per_token_head(128) == 139264
    assert bench.decode_bytes_per_head(128, 128, 2) == 132868
