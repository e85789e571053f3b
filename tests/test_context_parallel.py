"""Exchange logic of the time-axis split (context parallelism), on CPU with gloo.

The per-segment steps are replaced by stand-ins built on the fp64 oracle (a
segment's run from a state, its transfer as the run of the identity state with
zero values); what is under test is the orchestration: which rank starts from
the sequence's initial state, the one all-gather, the fold over the earlier
segments and the correction.  Concatenated over ranks, the outputs and the last
rank's final state must equal the oracle's run of the whole sequence.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NAMES = ("q", "k", "v", "log_alpha", "beta")
B, T, H, D = 2, 90, 2, 16


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs():
    from gated_delta_rule_109_b200 import inputs as I
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=B, H=H, T=T, dk=D, dv=D, dtype="f32", seed=901)
    return I.make_inputs(w, "cpu")


def _cuts(world):
    return [round(T * r / world) for r in range(world + 1)]


def _oracle_ops():
    import types
    import oracle

    def run(seg, v, s0):
        o, s = oracle.forward(seg["q"], seg["k"], v, seg["log_alpha"], seg["beta"], s0)
        return torch.from_numpy(o), torch.from_numpy(s)

    def segment_local(q, k, v, la, beta, s0, ws):
        ws.update(q=q, k=k, log_alpha=la, beta=beta, zero=torch.zeros_like(v))
        out, lf = run(ws, v, s0)
        eye = torch.eye(D, dtype=torch.float64).expand(B, H, D, D).contiguous()
        _, P = run(ws, ws["zero"], eye)
        return out, lf, P

    def segment_start_state(P, F):
        s = F[0]
        for j in range(1, P.shape[0]):
            s = F[j] + P[j] @ s
        return s

    def segment_correct(start, lf, out, ws):
        o, s = run(ws, ws["zero"], start)
        out += o
        return lf + s

    return types.SimpleNamespace(segment_local=segment_local, segment_start_state=segment_start_state,
                                 segment_correct=segment_correct)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        from gated_delta_rule_109_b200 import context_parallel as cp
        x = _inputs()
        a, b = _cuts(world)[rank:rank + 2]
        seg = [x[n][:, a:b].contiguous() for n in NAMES]
        out, final = cp.forward_context_parallel(*seg, x["initial_state"], workspace={}, ops=_oracle_ops())
        q.put((rank, out.numpy(), final.numpy()))
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_time_split_across_ranks_equals_whole_sequence(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=200) for _ in procs], key=lambda t: t[0])
    for p in procs:
        p.join(timeout=30)
    assert all(not isinstance(r[1], str) for r in res), res
    import oracle
    x = _inputs()
    o_ref, s_ref = oracle.forward(*(x[n] for n in NAMES), x["initial_state"])
    out = np.concatenate([r[1] for r in res], axis=1)
    assert out.shape == o_ref.shape
    np.testing.assert_allclose(out, o_ref, rtol=0, atol=1e-9 * np.abs(o_ref).max())
    np.testing.assert_allclose(res[-1][2], s_ref, rtol=0, atol=1e-9 * np.abs(s_ref).max())
    # every rank's final is the true state at the end of its segment
    cuts = _cuts(world)
    for r in range(world - 1):
        _, s_r = oracle.forward(*(x[n][:, :cuts[r + 1]] for n in NAMES), x["initial_state"])
        np.testing.assert_allclose(res[r][2], s_r, rtol=0, atol=1e-9 * np.abs(s_r).max())


def test_single_rank_is_the_local_run():
    """World size 1 (a one-process gloo group): no fold, no correction."""
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=30))
    try:
        from gated_delta_rule_109_b200 import context_parallel as cp
        import oracle
        x = _inputs()
        out, final = cp.forward_context_parallel(*(x[n] for n in NAMES), x["initial_state"], workspace={},
                                                 ops=_oracle_ops())
        o_ref, s_ref = oracle.forward(*(x[n] for n in NAMES), x["initial_state"])
        assert np.array_equal(out.numpy(), o_ref) and np.array_equal(final.numpy(), s_ref)
    finally:
        dist.destroy_process_group()
