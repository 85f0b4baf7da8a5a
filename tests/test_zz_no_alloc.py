"""The allocation-free GEMM entry point, checked against the oracle and against the
workspace-taking entry point.

apex_w4a4_gemm_noalloc serves callers that cannot allocate device memory while they run
(runtimes that budget every device byte in advance, plugin hosts whose allocator is off
limits, latency-critical paths that must avoid cudaMalloc/cudaFree stalls).  Its split-K
scratch is a fixed array inside the library, shared by every call on a device, so two
calls in a row also check that the second one does not see the first one's leftovers.
Both entry points take the same work plan and the same fixed-order split-K reduction, so
their outputs must be bit-identical, not merely close.

This file is collected last, so a run that stops at its first failure has already run
every other test; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest

import oracle
from group_quantized_w4a4_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def apex():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_quantized_w4a4_b200 as m
    m.load_library()
    return m


def operands(apex, M, N, K, gw, seed):
    """GPU-quantized operands, checked bit for bit against the oracle's quantizer, and the
    oracle's fp64 GEMM of them."""
    a = synth.activations(M, K, "normal", seed + M)
    w = synth.weights(N, K, seed + N)
    ap, sa = apex.quantize_act(torch.from_numpy(a).cuda(), 128)
    wp, sw = apex.pack_weights(torch.from_numpy(w).cuda(), gw)
    torch.cuda.synchronize()
    ap_ref, sa_ref = oracle.quantize_pack(a, 128)
    wp_ref, sw_ref = oracle.quantize_pack(w, gw)
    assert np.array_equal(ap.cpu().numpy(), ap_ref)
    assert np.array_equal(wp.cpu().numpy(), wp_ref)
    assert np.array_equal(sa.cpu().numpy().view(np.uint16), sa_ref.view(np.uint16))
    assert np.array_equal(sw.cpu().numpy().view(np.uint16), sw_ref.view(np.uint16))
    ref = oracle.gemm(ap_ref, sa_ref, wp_ref, sw_ref, M, N, K, 128, gw)
    return (ap, sa, wp, sw), ref


# (16, 16384, 8192): 128 tiles on 148 SMs, a true stream-K plan in which CTAs hold pieces of
# two tiles and use the shared arrival counters for both; (16, 2048, 8192): every tile split
# 9 ways through global memory; (32, 1024, 4096, 512): coarse weight groups; (16, 256, 512):
# whole tiles, no scratch at all.
@pytest.mark.parametrize("M,N,K,gw", [(16, 16384, 8192, 128), (16, 2048, 8192, 128),
                                      (32, 1024, 4096, 512), (16, 256, 512, 128)])
def test_noalloc_matches_oracle_and_workspace_gemm_twice(apex, M, N, K, gw):
    (ap, sa, wp, sw), ref = operands(apex, M, N, K, gw, 70)
    ws = apex.workspace(M, N, K, 128, gw)
    y_ws = torch.empty((M, N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm(M, N, K, 128, gw, ap, sa, wp, sw, y_ws, ws)
    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        apex.apex_w4a4_gemm_noalloc(M, N, K, 128, gw, ap, sa, wp, sw, y)
        outs.append(y)
    torch.cuda.synchronize()
    assert apex.apex_get_device_status() == 0
    ok, ratio = oracle.within_tolerance(y_ws.cpu().numpy().astype(np.float64), ref)
    assert ok, f"apex_w4a4_gemm outside tolerance (worst err/bound {ratio:.3f})"
    for y in outs:
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), \
            "no-alloc output is not bit-identical to apex_w4a4_gemm"
        ok, ratio = oracle.within_tolerance(y.cpu().numpy().astype(np.float64), ref)
        assert ok, f"no-alloc output outside tolerance (worst err/bound {ratio:.3f})"


def test_noalloc_recovers_after_a_timed_out_call(apex):
    # A call whose pipeline gives up (one bulk copy withheld, 50 ms wait limit) leaves its
    # split-K counters wherever it stopped; the next call clears them and is exact again.
    M, N, K = 16, 2048, 8192
    (ap, sa, wp, sw), ref = operands(apex, M, N, K, 128, 80)
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    apex.apex_set_wait_limit_ns(50_000_000)
    try:
        apex.apex_debug_withhold_step(1)
        apex.apex_w4a4_gemm_noalloc(M, N, K, 128, 128, ap, sa, wp, sw, y)
        assert apex.apex_get_device_status() == apex.APEX_ERR_TIMEOUT
    finally:
        apex.apex_debug_withhold_step(-1)
        apex.apex_set_wait_limit_ns(2_000_000_000)
    y2 = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_noalloc(M, N, K, 128, 128, ap, sa, wp, sw, y2)
    torch.cuda.synchronize()
    assert apex.apex_get_device_status() == 0
    ok, ratio = oracle.within_tolerance(y2.cpu().numpy().astype(np.float64), ref)
    assert ok, f"call after the timeout outside tolerance (worst err/bound {ratio:.3f})"


def test_noalloc_refuses_problems_beyond_its_scratch(apex):
    # A problem whose split-K scratch exceeds the fixed array is refused before launch.
    M, N, K = 128, 8192, 8192          # split in two: 2 x 128 x 8192 fp32 partials + counters
    need = apex.apex_w4a4_gemm_workspace_size(M, N, K, 128, 128)
    if need <= (8 << 20):
        pytest.skip("this problem needs no more scratch than the fixed array holds")
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_noalloc(M, N, K, 128, 128, dummy, dummy, dummy, dummy, dummy)
    assert e.value.code == apex.APEX_ERR_UNSUPPORTED
