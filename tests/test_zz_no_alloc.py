"""lcla_forward_noalloc: the forward for callers that cannot allocate.

Some callers of this library cannot obtain device scratch memory -- a plugin
whose host application owns every device allocation through its own pool, or
a real-time loop that must not enter cudaMalloc/cudaFree (they can block and
synchronise the device).  lcla_forward_noalloc serves them from a scratch
array compiled into the library.  These tests call it through the C ABI
(ctypes, raw device pointers) twice in a row and check each result against
lcla_forward with a caller-allocated workspace, within the parity tolerance
the other tests use.  This file is named to be collected last.
"""
import ctypes

import pytest
import torch

import block_causal_relu_b200 as lcla
from gpu_util import host, inputs_to_dev
from parity import check_outputs, check_state
from workloads import NAMED, Spec, make_inputs

pytestmark = pytest.mark.gpu

NOALLOC_SCRATCH_BYTES = 64 << 20
TOO_LARGE = 6


def _fn():
    f = lcla.lib.lcla_forward_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [P, P, P, P, P, I, I, I, I, I, F, P, P, I, P]
    f.restype = I
    return f


def call_noalloc(q, k, v, c, s, block_len, eps, out, state):
    B, N, H, d = q.shape
    code = lcla.BF16 if q.dtype == torch.bfloat16 else lcla.F32
    return _fn()(q.data_ptr(), k.data_ptr(), v.data_ptr(), c.data_ptr(), s.data_ptr(), B, H, N, d,
                 block_len, eps, out.data_ptr(), state.data_ptr(), code,
                 torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("spec", [
    NAMED["fwd480p_bf16"],                                                   # tensor-core path
    Spec("noalloc_f32", 2, 5, 3001, 32, 700, "f32", 41, qk_dist="laplace_negrows", v_sigma=2.0),
    Spec("noalloc_chunk", 1, 4, 5000, 32, 7, "bf16", 42),                    # chunk mode
], ids=lambda s: s.name)
def test_noalloc_matches_forward_twice(spec):
    assert lcla.forward_workspace_bytes(spec.B, spec.H, spec.N, 32, spec.block_len,
                                        0 if spec.dtype == "bf16" else 1) <= NOALLOC_SCRATCH_BYTES
    inp = make_inputs(spec)
    q, k, v, c, s = inputs_to_dev(inp)
    ref, ref_st = lcla.forward(q, k, v, c, s, spec.block_len, spec.eps)
    torch.cuda.synchronize()
    for attempt in range(2):
        out = torch.full_like(q, float("nan"))
        st = torch.full((spec.B, spec.H, 33, 32), float("nan"), device="cuda")
        rc = call_noalloc(q, k, v, c, s, spec.block_len, spec.eps, out, st)
        assert rc == 0, lcla.lib.lcla_status_string(rc)
        torch.cuda.synchronize()
        check_outputs(host(out), host(ref), spec.dtype, f"noalloc call {attempt}", ulps=1.0)
        check_state(host(st), host(ref_st), f"noalloc state call {attempt}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # about 2 GB of segment states: far beyond the built-in array; nothing is touched
    B, H, N, L = 1, 16, 1 << 20, 65
    assert lcla.forward_workspace_bytes(B, H, N, 32, L, lcla.BF16) > NOALLOC_SCRATCH_BYTES
    a = 1 << 20
    rc = _fn()(a, 2 * a, 3 * a, 4 * a, 5 * a, B, H, N, 32, L, 1e-8, 6 * a, 7 * a, lcla.BF16, None)
    assert rc == TOO_LARGE
    assert b"scratch" in lcla.lib.lcla_status_string(rc)
