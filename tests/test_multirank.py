"""Host logic of the multi-GPU benchmark path, on CPU with gloo, world size 2.

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


@pytest.mark.timeout(180)
def test_two_rank_weak_scaling_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=150) for _ in procs]
    for p in procs:
        p.join(timeout=30)
    assert all(len(x) == 6 for x in res), res
    res.sort()
    (r0, ws0, seed0, T0, mx0, _), (r1, ws1, seed1, T1, mx1, rc1) = res
    assert ws0 == ws1 == 2
    assert seed0 != seed1 and T0 == T1 == 65536      # independent batches of the same size
    assert mx0 == mx1 == 15.0                          # max over ranks
    assert rc1 == 0                                    # reference arm: rank 1 does no work


def test_single_process_helpers_are_identities():
    import bench
    from gated_delta_rule_109_b200 import inputs as I
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.rank_workload(I.PREFILL_H32_T64K, 0).seed == I.PREFILL_H32_T64K.seed
    assert bench.prefill_bytes_per_token_head(128, 128, 2) == 1796
    assert bench.prefill_flops_per_token_head(128) == 139264
    assert bench.decode_bytes_per_head(128, 128, 2) == 132868
