"""The library's calls captured in a CUDA graph.

Every call enqueues its work on the caller's stream and allocates nothing, so
a loop of forwards or streaming steps can be captured once and replayed; the
replay must give the same bits as the eager calls."""
import pytest
import torch

import block_causal_relu_b200 as lcla
from gpu_util import inputs_to_dev
from workloads import Spec, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,dtype", [(32, "bf16"), (64, "bf16"), (32, "f32")])
def test_step_sequence_graph_replay_matches_eager(d, dtype):
    L = 640
    spec = Spec("graph", 2, 6, 4 * L + 100, d, L, dtype, 2501, qk_dist="laplace_negrows", v_sigma=2.0)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    bounds = [(t, min(spec.N, t + L)) for t in range(0, spec.N, L)]
    blocks = [[x[:, t0:t1].contiguous() for x in (q, k, v)] + [c[t0:t1].contiguous(), s[t0:t1].contiguous()]
              for t0, t1 in bounds]
    code = lcla.BF16 if dtype == "bf16" else lcla.F32
    ws = torch.empty(max(1, lcla.step_workspace_bytes(spec.B, spec.H, L, d, code)), dtype=torch.uint8, device="cuda")
    state = torch.zeros((spec.B, spec.H, d + 1, d), device="cuda")
    outs = [torch.empty_like(b[0]) for b in blocks]

    def sequence(stream):
        state.zero_()
        for i, b in enumerate(blocks):
            lcla.step(*b, state, True, spec.eps, out=outs[i], workspace=ws, stream=stream)

    sequence(torch.cuda.current_stream())
    torch.cuda.synchronize()
    eager = [o.clone() for o in outs]
    eager_state = state.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        sequence(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        sequence(torch.cuda.current_stream())
    for o in outs:
        o.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, eager):
        assert torch.equal(a, b)
    assert torch.equal(state, eager_state)


def test_forward_graph_replay_matches_eager():
    spec = Spec("graphfwd", 1, 8, 5000, 32, 1200, "bf16", 2502)
    inp = make_inputs(spec, threads=2)
    q, k, v, c, s = inputs_to_dev(inp)
    ws = torch.empty(lcla.forward_workspace_bytes(1, 8, 5000, 32, 1200, lcla.BF16), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    st = torch.empty((1, 8, 33, 32), device="cuda")
    lcla.forward(q, k, v, c, s, 1200, spec.eps, out=out, state_out=st, workspace=ws)
    torch.cuda.synchronize()
    eager, eager_st = out.clone(), st.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        lcla.forward(q, k, v, c, s, 1200, spec.eps, out=out, state_out=st, workspace=ws, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lcla.forward(q, k, v, c, s, 1200, spec.eps, out=out, state_out=st, workspace=ws,
                     stream=torch.cuda.current_stream())
    out.zero_()
    st.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager) and torch.equal(st, eager_st)
