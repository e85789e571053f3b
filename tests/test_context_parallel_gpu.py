"""context_parallel.forward_context_parallel with the library's kernels, every
rank of a three-segment split emulated in one process on one device: the
torch.distributed calls are replaced by stand-ins that hand each "rank" the
(transfer, local final) pairs the real kernels produced for the other segments.
Nothing waits on another process; the exchange logic itself is covered under
gloo in test_context_parallel.py."""
import pytest
import torch

import gated_delta_rule_109_b200 as kda
import oracle
from gated_delta_rule_109_b200 import context_parallel as cp
from gated_delta_rule_109_b200 import inputs as I

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "log_alpha", "beta")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gated_delta_rule_109_b200 import build
    build.build()


def test_three_rank_split_with_kernel_ops(monkeypatch):
    w = I.scaled(I.PREFILL_B4_T16K_STATE, B=2, H=3, T=600, seed=9500)
    x = I.make_inputs(w, "cuda")
    cuts = [0, 200, 450, 600]
    R = len(cuts) - 1
    segs = [{n: x[n][:, cuts[r]:cuts[r + 1]].contiguous() for n in NAMES} for r in range(R)]
    wss = [kda.make_workspace(w.B, cuts[r + 1] - cuts[r], w.H, 128, 128, segment=True) for r in range(R)]
    pairs = []
    for r in range(R):
        _, lf, P = cp.KERNEL_OPS.segment_local(*(segs[r][n] for n in NAMES), x["initial_state"] if r == 0 else None,
                                               wss[r])
        pairs.append(torch.stack([P, lf]).contiguous())
    outs, finals = [], []
    for r in range(R):
        monkeypatch.setattr(cp.dist, "get_rank", lambda group=None, r=r: r)
        monkeypatch.setattr(cp.dist, "get_world_size", lambda group=None: R)

        def all_gather(out_list, t, group=None):
            assert torch.equal(t, pairs[len(outs)])          # this rank's own pair, as computed above
            for j in range(R):
                out_list[j].copy_(pairs[j])
        monkeypatch.setattr(cp.dist, "all_gather", all_gather)
        o, f = cp.forward_context_parallel(*(segs[r][n] for n in NAMES), x["initial_state"], workspace=wss[r])
        outs.append(o)
        finals.append(f)
    torch.cuda.synchronize()
    kda.check_status()
    o_ref, s_ref = oracle.forward(*(x[n] for n in NAMES), x["initial_state"])
    assert oracle.parity_error(torch.cat(outs, dim=1).cpu().numpy(), o_ref) <= 2e-3
    assert oracle.parity_error(finals[-1].cpu().numpy(), s_ref) <= 2e-3
    # every rank's final is the true state at the end of its segment
    for r in range(R - 1):
        _, s_r = oracle.forward(*(x[n][:, :cuts[r + 1]] for n in NAMES), x["initial_state"])
        assert oracle.parity_error(finals[r].cpu().numpy(), s_r) <= 2e-3
