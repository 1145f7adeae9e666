"""The C-ABI library on the host: it loads, exports every declared entry
point, answers workspace queries, and rejects invalid calls before touching
the GPU (every call here fails validation, so no kernel is launched)."""
import ctypes
import os
import re

import pytest

import block_causal_relu_b200 as lcla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA = range(6)


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lcla.h")).read()
    return sorted(set(re.findall(r"LCLA_API\s+[\w\s\*]+?\b(lcla_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"lcla_forward", "lcla_step", "lcla_forward_workspace_bytes",
            "lcla_step_workspace_bytes", "lcla_status_string", "lcla_version",
            "lcla_forward_blocks", "lcla_forward_blocks_workspace_bytes", "lcla_temporal_conv",
            "lcla_shard_begin", "lcla_shard_end", "lcla_shard_workspace_bytes",
            "lcla_selftest_bounded_wait"} <= set(names)
    lib = ctypes.CDLL(lcla.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version():
    for s in range(6):
        assert lcla.lib.lcla_status_string(s)
    assert b"unknown" in lcla.lib.lcla_status_string(99)
    assert lcla.lib.lcla_version() >= 100


def test_workspace_queries():
    f = lcla.forward_workspace_bytes
    assert f(1, 70, 32760, 32, 4680, lcla.BF16) > 0
    assert f(1, 70, 32760, 32, 4680, lcla.BF16) % 256 == 0
    assert f(1, 16, 65536, 32, 1, lcla.F32) > 0
    assert f(1, 1, 0, 32, 4, lcla.BF16) == 0          # empty sequence needs nothing
    assert f(0, 1, 10, 32, 4, lcla.BF16) == 0          # invalid -> 0
    assert f(1, 1, 10, 128, 4, lcla.BF16) == 0         # unsupported -> 0
    # head dim 64: block mode at every block length, states of 65 x 64 floats
    assert f(1, 35, 32760, 64, 4680, lcla.BF16) > 0
    assert f(1, 35, 32760, 64, 4680, lcla.BF16) % 256 == 0
    assert f(1, 2, 300, 64, 1, lcla.F32) >= 256 + 2 * 300 * 2 * 65 * 64 * 4   # partials and prefixes per block
    assert f(1, 70000, 10, 64, 4, lcla.BF16) == 0       # grid y limit of the d = 64 kernels
    info = lcla.plan_info(1, 35, 32760, 64, 4680, lcla.BF16)
    assert not info["chunk_mode"] and info["tensor_cores"]          # bf16: two heads per tensor-core unit
    assert not lcla.plan_info(1, 35, 32760, 64, 4680, lcla.F32)["tensor_cores"]   # fp32: CUDA cores
    assert not lcla.plan_info(1, 2, 300, 64, 1, lcla.F32)["chunk_mode"]
    assert f(1, 1, 10, 32, 0, lcla.BF16) == 0
    assert f(1, 1, 10, 32, 4, 7) == 0
    # independent of anything but the arguments
    assert f(2, 70, 63960, 32, 4680, 0) == f(2, 70, 63960, 32, 4680, 0)
    assert lcla.step_workspace_bytes(2, 70, 4680, 32, lcla.BF16) > 0
    assert lcla.step_workspace_bytes(2, 70, 0, 32, lcla.BF16) == 0


A = 1 << 20   # fake, 16-byte aligned "device" addresses: validation never dereferences


def fwd(**kw):
    args = dict(q=A, k=2 * A, v=3 * A, c=4 * A, s=5 * A, B=1, H=2, N=100, d=32, L=10, eps=1e-8,
                out=6 * A, st=7 * A, dtype=0, ws=8 * A, wsb=1 << 20, stream=None)
    args.update(kw)
    return lcla.lib.lcla_forward(args["q"], args["k"], args["v"], args["c"], args["s"], args["B"],
                                 args["H"], args["N"], args["d"], args["L"], args["eps"],
                                 args["out"], args["st"], args["dtype"], args["ws"], args["wsb"],
                                 args["stream"])


def stp(**kw):
    args = dict(q=A, k=2 * A, v=3 * A, c=4 * A, s=5 * A, B=1, H=2, L=100, d=32, eps=1e-8,
                st=7 * A, save=1, out=6 * A, dtype=0, ws=8 * A, wsb=1 << 20, stream=None)
    args.update(kw)
    return lcla.lib.lcla_step(args["q"], args["k"], args["v"], args["c"], args["s"], args["B"],
                              args["H"], args["L"], args["d"], args["eps"], args["st"], args["save"],
                              args["out"], args["dtype"], args["ws"], args["wsb"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), INVALID), (dict(k=None), INVALID), (dict(v=None), INVALID),
    (dict(c=None), INVALID), (dict(s=None), INVALID), (dict(out=None), INVALID),
    (dict(N=-1), INVALID), (dict(B=0), INVALID), (dict(H=0), INVALID), (dict(B=-3), INVALID),
    (dict(L=0), INVALID), (dict(L=-5), INVALID), (dict(d=0), INVALID), (dict(d=31), INVALID),
    (dict(d=128), UNSUPPORTED), (dict(d=16), UNSUPPORTED), (dict(N=(1 << 30) + 1), UNSUPPORTED),
    (dict(dtype=2), INVALID), (dict(dtype=-1), INVALID),
    (dict(eps=-1.0), INVALID), (dict(eps=float("nan")), INVALID), (dict(eps=float("inf")), INVALID),
    (dict(q=A + 8), MISALIGNED), (dict(k=2 * A + 4), MISALIGNED), (dict(v=3 * A + 2), MISALIGNED),
    (dict(c=4 * A + 8), MISALIGNED), (dict(out=6 * A + 1), MISALIGNED), (dict(st=7 * A + 4), MISALIGNED),
    (dict(ws=8 * A + 8), MISALIGNED),
    (dict(ws=None), WORKSPACE), (dict(wsb=16), WORKSPACE),
    (dict(out=A), INVALID), (dict(out=2 * A + 64), INVALID), (dict(out=3 * A - 64), INVALID),
    (dict(out=4 * A), INVALID), (dict(out=7 * A), INVALID), (dict(out=8 * A + 4096), INVALID),
    (dict(ws=A), INVALID), (dict(st=A + 256), INVALID),
])
def test_forward_rejects(kw, code):
    assert fwd(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(st=None), INVALID), (dict(q=None), INVALID), (dict(L=-1), INVALID), (dict(B=0), INVALID),
    (dict(d=128), UNSUPPORTED), (dict(dtype=5), INVALID), (dict(st=7 * A + 8), MISALIGNED),
    (dict(ws=None), WORKSPACE), (dict(out=3 * A), INVALID), (dict(st=5 * A), INVALID),
    (dict(eps=-0.5), INVALID),
])
def test_step_rejects(kw, code):
    assert stp(**kw) == code


def test_trivial_calls_need_no_gpu():
    # an empty block is a valid no-op and touches nothing
    assert stp(L=0, q=None, k=None, v=None, c=None, s=None, out=None, ws=None, wsb=0) == OK


def test_explicit_blocks_workspace_and_arguments():
    f = lcla.forward_blocks_workspace_bytes
    # the same cut as uniform blocks of the mean length
    assert f(1, 70, 32760, 32, 7, lcla.BF16) == lcla.forward_workspace_bytes(1, 70, 32760, 32, 4680, lcla.BF16)
    assert f(1, 4, 100, 32, 0, lcla.BF16) == 0          # no blocks
    assert f(1, 4, 100, 32, 101, lcla.BF16) == 0        # more blocks than tokens
    assert f(1, 4, 100, 32, 3, lcla.BF16) > 0
    assert f(1, 4, 100, 128, 3, lcla.BF16) == 0         # d = 128 not served
    import ctypes
    a = 1 << 20
    fn = lcla.lib.lcla_forward_blocks
    # argument errors return before any launch (no device memory is touched)
    rc = fn(a, 2 * a, 3 * a, 4 * a, 5 * a, 1, 4, 100, 32, None, 3, 1e-8, 6 * a, None, lcla.BF16, None, 0, None)
    assert rc == 1                                      # offsets missing
    rc = fn(a, 2 * a, 3 * a, 4 * a, 5 * a, 1, 4, 100, 32, 7 * a + 2, 3, 1e-8, 6 * a, None, lcla.BF16, None, 0, None)
    assert rc == 3                                      # offsets not 4-byte aligned
    rc = fn(a, 2 * a, 3 * a, 4 * a, 5 * a, 1, 4, 100, 32, 7 * a, 101, 1e-8, 6 * a, None, lcla.BF16, None, 0, None)
    assert rc == 1                                      # more blocks than tokens
    rc = fn(a, 2 * a, 3 * a, 4 * a, 5 * a, 1, 4, 100, 32, 7 * a, 3, 1e-8, 6 * a, None, lcla.BF16, None, 0, None)
    assert rc == 4                                      # workspace missing


def test_temporal_conv_arguments():
    fn = lcla.lib.lcla_temporal_conv
    a = 1 << 20
    # argument errors return before any launch (no device memory is touched)
    assert fn(a, 1, 2, 3, 12, 2 * a, None, None, 0, 3 * a, lcla.BF16, None) == 1   # C not a multiple of 8
    assert fn(a, 1, 2, 3, 16, 2 * a, None, None, 0, 3 * a, 7, None) == 1            # bad dtype
    assert fn(a + 8, 1, 2, 3, 16, 2 * a, None, None, 0, 3 * a, lcla.BF16, None) == 3   # misaligned x
    assert fn(a, 1, 2, 3, 16, 2 * a, None, a + 64, 0, 3 * a, lcla.BF16, None) == 1     # cache inside x
    assert fn(a, 1, 0, 3, 16, 2 * a, None, None, 0, 3 * a, lcla.BF16, None) == 0       # no frames: nothing to do
    assert fn(None, 1, 2, 3, 16, 2 * a, None, None, 0, 3 * a, lcla.BF16, None) == 1    # x missing


def test_shard_workspace_and_arguments():
    f = lcla.shard_workspace_bytes
    # the forward's workspace plus one [B, H, d+1, d] fp32 carry slice
    assert f(1, 70, 18720, 32, 4680, lcla.BF16) == \
        lcla.forward_workspace_bytes(1, 70, 18720, 32, 4680, lcla.BF16) + 70 * 33 * 32 * 4
    assert f(1, 4, 0, 32, 16, lcla.BF16) == 0            # an empty shard needs nothing
    assert f(1, 4, 100, 128, 16, lcla.BF16) == 0         # d = 128 not served
    a = 1 << 20
    begin, end = lcla.lib.lcla_shard_begin, lcla.lib.lcla_shard_end
    # argument errors return before any launch (no device memory is touched)
    assert begin(a, 2 * a, 3 * a, 4 * a, 1, 4, 100, 32, 16, None, 0, 8 * a, 1 << 20, None) == INVALID
    assert begin(a, 2 * a, 3 * a, 4 * a, 1, 4, 100, 32, 16, 5 * a + 4, 0, 8 * a, 1 << 20, None) == MISALIGNED
    assert begin(a, 2 * a, 3 * a, 4 * a, 1, 4, 100, 32, 16, 5 * a, 0, None, 0, None) == WORKSPACE
    assert begin(a, 2 * a, 3 * a, 4 * a, 1, 4, 100, 32, 16, a + 64, 0, 8 * a, 1 << 20, None) == INVALID  # total in k
    assert begin(None, 2 * a, 3 * a, 4 * a, 1, 4, 100, 32, 16, 5 * a, 0, 8 * a, 1 << 20, None) == INVALID
    assert begin(a, 2 * a, 3 * a, 4 * a, 1, 4, 100, 48, 16, 5 * a, 0, 8 * a, 1 << 20, None) == UNSUPPORTED

    def e(**kw):
        args = dict(q=a, k=2 * a, v=3 * a, c=4 * a, s=5 * a, B=1, H=4, N=100, d=32, L=16, eps=1e-8,
                    tot=6 * a, R=2, r=1, sin=None, out=7 * a, sout=None, dtype=0, ws=8 * a, wsb=1 << 20)
        args.update(kw)
        return end(*args.values(), None)
    assert e(R=0, r=0) == INVALID                        # no ranks
    assert e(r=2) == INVALID                             # rank out of range
    assert e(r=-1) == INVALID
    assert e(tot=None) == INVALID                        # totals missing
    assert e(tot=6 * a + 8) == MISALIGNED
    assert e(eps=-1.0) == INVALID
    assert e(sout=6 * a + 256) == INVALID                # final state inside the totals
    assert e(sin=9 * a, sout=9 * a + 128) == INVALID     # partial overlap of state_in and state_out
    assert e(ws=None, wsb=0) == WORKSPACE
    assert e(out=6 * a) == INVALID                       # out over the totals


def test_selftest_arguments():
    fn = lcla.lib.lcla_selftest_bounded_wait
    assert fn(1, None, None) == INVALID
    assert fn(1, (1 << 20) + 4, None) == MISALIGNED


def test_header_compiles_as_c_and_a_c_program_links(tmp_path):
    """The boundary is plain C: the header compiles as pedantic C99 and a C
    program links against the library and calls it (the planner touches no
    device)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text('#include "lcla.h"\n'
                   "int main(void) {\n"
                   "    int info[5];\n"
                   "    if (lcla_forward_plan_info(1, 70, 32760, 32, 4680, LCLA_BF16, info) != LCLA_OK) return 1;\n"
                   "    if (info[0] != 0 || info[4] != 1) return 2;\n"
                   "    if (lcla_forward_workspace_bytes(1, 70, 32760, 64, 4680, LCLA_BF16) == 0) return 3;\n"
                   "    return lcla_version() >= 100 ? 0 : 4;\n"
                   "}\n")
    libdir = os.path.dirname(lcla.LIB_PATH)
    exe = tmp_path / "abi"
    subprocess.check_call([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-L", libdir, "-llcla", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    assert subprocess.run([str(exe)]).returncode == 0
