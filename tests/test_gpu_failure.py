"""The failure path of the bounded waits, on the GPU, without a fault: a wait on an mbarrier
that nothing completes, and the acceptance draw kernel's wait on a sequence flag that nothing
raises, each give up after their poll limit, report the wait-timeout bit in the status word
and return; the context stays usable (a verify call after them is still exact)."""
import pytest
import torch

from gated_deltanet_mixer_verify_b200.inputs import make_inputs, workload
from gdn_helpers import TOL, gpu_verify, oracle_verify, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn(cuda_device):
    from gated_deltanet_mixer_verify_b200 import build, gdn as g
    build.build()
    return g


def test_bounded_wait_reports_timeout_and_context_survives(gdn):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    gdn.selftest_bounded_wait(status, polls=1024)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    # the context still computes: a verify call afterwards matches the oracle
    w = workload("batched_verify", B=2, seed=95)
    x = make_inputs(w)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, S = gpu_verify(gdn, to_dev(x), x["accept_len"].numpy(), status=st2)
    o_ref, S_ref, _ = oracle_verify(x, x["accept_len"].numpy())
    assert rel_err(o, o_ref) <= TOL and rel_err(S, S_ref) <= TOL and int(st2.item()) == 0


def test_accept_flag_wait_reports_timeout_and_context_survives(gdn):
    # The acceptance draw kernel alone, its sequence's flag never raised: every CTA gives up,
    # reports the wait-timeout bit and writes next token 0; nothing else is touched.
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nt = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    gdn.selftest_accept_wait(status, nt, polls=256)
    torch.cuda.synchronize()
    assert int(status.item()) == 2 and int(nt.item()) == 0
    # the context still computes: a verify call afterwards matches the oracle
    w = workload("batched_verify", B=2, seed=96)
    x = make_inputs(w)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, S = gpu_verify(gdn, to_dev(x), x["accept_len"].numpy(), status=st2)
    o_ref, S_ref, _ = oracle_verify(x, x["accept_len"].numpy())
    assert rel_err(o, o_ref) <= TOL and rel_err(S, S_ref) <= TOL and int(st2.item()) == 0
