"""Failure detection without a GPU fault.

The tensor-core kernels bound every mbarrier wait (1 s of globaltimer); a wait
that gives up raises the CTA's abort flag instead of hanging.  The self-test
runs that wait on a barrier nothing arrives at: it must give up after about
its limit and report it, and the context must stay usable -- a forward right
after it matches the oracle and leaves a zero device status.  The control run
completes the barrier first and must pass straight through."""
import pytest
import torch

import block_causal_relu_b200 as lcla
import oracle
from gpu_util import host, inputs_to_dev
from parity import check_outputs
from workloads import Spec, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_completes_when_the_phase_completes():
    gave_up, ns, flag = lcla.selftest_bounded_wait(True)
    assert not gave_up and flag == 0
    assert ns < 50_000_000


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    gave_up, ns, flag = lcla.selftest_bounded_wait(False)
    assert gave_up and flag == 1
    assert 0.9e9 <= ns <= 5e9, ns
    # the device still works: a forward, its status word and its outputs
    spec = Spec("after", 1, 4, 1500, 32, 500, "bf16", 2601)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    ws = torch.empty(lcla.forward_workspace_bytes(1, 4, 1500, 32, 500, lcla.BF16), dtype=torch.uint8, device="cuda")
    out, _ = lcla.forward(q, k, v, c, s, 500, spec.eps, workspace=ws)
    torch.cuda.synchronize()
    assert lcla.device_status(ws) == 0
    ref, _, _ = oracle.recurrence(inp.q, inp.k, inp.v, inp.rope_cos, inp.rope_sin, 500, spec.eps)
    check_outputs(host(out), ref, "bf16", "forward after a timed-out wait")
