"""gmm_fwd_noalloc: the forward gmm for callers that cannot allocate device
memory (code under a runtime or framework that owns all device memory and
forbids allocations after start-up, or that cannot afford the device
synchronization of cudaMalloc / cudaFree).  Its scratch is a fixed array
inside the library instead of a caller-provided workspace.

Called through the C-ABI on two calls in a row with different inputs, so that
the second call cannot pass on what the first left in the shared array.  Each
output is checked against the oracle within the parity tolerance, and bit for
bit against gmm_fwd (the entry point that takes a workspace: the same kernels
on the same inputs, so any difference would come from the shared array).
Device-detected errors are read back with gmm_fwd_noalloc_status.  This file
sorts last so that a run stopping at the first failure has run every other
test; it depends on no other test.
"""
import ctypes

import pytest
import torch

import moe_fp8_grouped_b200 as gm
import oracle
from moe_fp8_grouped_b200 import _binding as B
from moe_fp8_grouped_b200 import synth
from parity import assert_close

pytestmark = pytest.mark.gpu


def _noalloc_fwd(lhs, codes, scales, gs, rule, s, out):
    stream = torch.cuda.current_stream().cuda_stream
    a = B.Operand(lhs.data_ptr(), B.DT_BF16, s.data_ptr() if s is not None else None,
                  B.Q_STATIC if rule == "static" else B.Q_DYNAMIC)
    b = B.Operand(codes.data_ptr(), B.DT_E4M3, scales.data_ptr(), B.Q_NONE)
    M, K = lhs.shape
    G, _, N = codes.shape
    return B.lib().gmm_fwd_noalloc(a, b, 0, gs.data_ptr(), G, M, K, N, out.data_ptr(),
                                   B.DT_F32 if out.dtype == torch.float32 else B.DT_BF16, stream)


def _noalloc_status():
    bits = ctypes.c_uint32(0xFFFFFFFF)
    st = B.lib().gmm_fwd_noalloc_status(ctypes.byref(bits), torch.cuda.current_stream().cuda_stream)
    return st, bits.value


@pytest.mark.parametrize("rule", ["static", "dynamic"])
def test_noalloc_matches_oracle_and_gmm_fwd_on_two_calls(rule):
    dev = torch.device("cuda:0")
    cases = [synth.small_case(5, 700, 384, 640, seed=21, sizes=[1, 129, 0, 300, 200]),
             synth.small_case(3, 1000, 512, 256, seed=22, sizes=[400, 350, 250])]
    for inp in cases:
        lhs, w, gs = inp.lhs.to(dev), inp.w.to(dev), inp.group_sizes.to(dev)
        s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
        sarg = s if rule == "static" else None
        codes, scales = gm.gmm_quantize_rhs(w)
        M, N = lhs.shape[0], w.shape[2]
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device=dev)
        assert _noalloc_fwd(lhs, codes, scales, gs, rule, sarg, out) == 0
        assert _noalloc_status() == (0, 0)  # synchronizes the stream
        qr, sr = oracle.quantize_rhs(inp.w)
        ref, ab = oracle.gmm_fwd(inp.lhs, oracle.Q_STATIC if rule == "static" else oracle.Q_DYNAMIC,
                                 inp.static_scale, qr, sr, inp.group_sizes)
        assert_close(out, ref, ab, f"noalloc vs oracle ({rule})")
        same = gm.gmm_fwd(lhs, codes, scales, gs, rule=rule, static_scale=sarg, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert torch.equal(out, same), f"noalloc differs from gmm_fwd ({rule})"


def test_noalloc_status_reports_bad_group_sizes_then_clears():
    dev = torch.device("cuda:0")
    inp = synth.small_case(3, 300, 256, 256, seed=23, sizes=[100, 150, 50])
    lhs, w = inp.lhs.to(dev), inp.w.to(dev)
    codes, scales = gm.gmm_quantize_rhs(w)
    s = torch.tensor([inp.static_scale], dtype=torch.float32, device=dev)
    out = torch.empty((300, 256), dtype=torch.bfloat16, device=dev)
    bad = torch.tensor([200, 150, 50], dtype=torch.int32, device=dev)  # sums past M: clamped on the device
    assert _noalloc_fwd(lhs, codes, scales, bad, "static", s, out) == 0
    st, bits = _noalloc_status()
    assert st == 7 and bits & B.DEV_GROUP_SIZES  # GMM_ERR_GROUP_SIZES
    good = inp.group_sizes.to(dev)
    assert _noalloc_fwd(lhs, codes, scales, good, "static", s, out) == 0
    assert _noalloc_status() == (0, 0)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    dev = torch.device("cuda:0")
    M, K, N, G = 8192, 8192, 256, 4  # needs more than 32 MiB of scratch
    assert gm.gmm_workspace_bytes(0, M, K, N, G) > (32 << 20)
    lhs = torch.zeros((M, K), dtype=torch.bfloat16, device=dev)
    codes = torch.zeros((G, K, N), dtype=torch.uint8, device=dev)
    scales = torch.ones((G, N), dtype=torch.float32, device=dev)
    gs = torch.full((G,), M // G, dtype=torch.int32, device=dev)
    out = torch.zeros((M, N), dtype=torch.bfloat16, device=dev)
    s = torch.tensor([1.0], dtype=torch.float32, device=dev)
    assert _noalloc_fwd(lhs, codes, scales, gs, "static", s, out) == 9  # GMM_ERR_WORKSPACE
