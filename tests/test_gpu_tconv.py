"""lcla_temporal_conv on the GPU against the fp64 oracle, its save semantics
and streaming over blocks of frames."""
import numpy as np
import pytest
import torch

import block_causal_relu_b200 as lcla
from gpu_util import host
from oracle.tconv import temporal_conv
from parity import check_outputs
from workloads import f64_to_bf16_bits

pytestmark = pytest.mark.gpu


def _inputs(seed, B, F, S, C, dtype, with_cache, with_bias):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, F * S, C))
    cache = rng.standard_normal((B, S, C)) if with_cache else None
    w = rng.standard_normal((2, C)).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32) if with_bias else None
    if dtype == "bf16":
        xh = f64_to_bf16_bits(x).reshape(x.shape)
        ch = None if cache is None else f64_to_bf16_bits(cache).reshape(cache.shape)
    else:
        xh = x.astype(np.float32)
        ch = None if cache is None else cache.astype(np.float32)
    return xh, ch, w, b


def _dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


CASES = [  # (B, F, S, C, dtype, with_cache, with_bias)
    (2, 5, 123, 64, "bf16", True, True),
    (2, 5, 123, 64, "f32", False, True),
    (1, 3, 7, 8, "f32", True, False),
    (3, 1, 50, 136, "bf16", True, True),
    (1, 21, 30 * 52, 2240, "bf16", True, True),      # the 480p-like latent: 21 frames of 30 x 52, width 2240
]


@pytest.mark.parametrize("B,F,S,C,dtype,with_cache,with_bias", CASES)
def test_against_oracle(B, F, S, C, dtype, with_cache, with_bias):
    x, cache, w, b = _inputs(100 + F + C, B, F, S, C, dtype, with_cache, with_bias)
    xd, cd = _dev(x), _dev(cache)
    y = lcla.temporal_conv(xd, S, _dev(w), _dev(b), cd, save=True)
    torch.cuda.synchronize()
    ref, last = temporal_conv(x, S, w, b, cache)
    check_outputs(host(y), ref, dtype, f"temporal conv {B}x{F}x{S}x{C} {dtype}")
    if cd is not None:   # the saved frame is x's last frame, bit for bit
        assert torch.equal(cd, xd[:, -S:]), "saved cache differs from the last frame"


def test_save_flag_and_streaming():
    B, F, S, C = 2, 9, 64, 256
    x, cache, w, b = _inputs(7, B, F, S, C, "bf16", True, True)
    xd, wd, bd = _dev(x), _dev(w), _dev(b)
    c0 = _dev(cache)
    keep = c0.clone()
    y_a = lcla.temporal_conv(xd, S, wd, bd, c0, save=False)
    y_b = lcla.temporal_conv(xd, S, wd, bd, c0, save=False)
    torch.cuda.synchronize()
    assert torch.equal(c0, keep), "save=0 wrote the cache"
    assert torch.equal(y_a, y_b), "repeated save=0 calls differ"
    # three blocks of 3 frames, each saving its last frame, equal one call over all 9 frames
    whole = lcla.temporal_conv(xd, S, wd, bd, keep.clone(), save=False)
    c = keep.clone()
    parts = [lcla.temporal_conv(xd[:, i * 3 * S:(i + 1) * 3 * S].contiguous(), S, wd, bd, c, save=True)
             for i in range(3)]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), whole), "block-by-block differs from one call"
    assert torch.equal(c, xd[:, -S:]), "cache after the last block"
