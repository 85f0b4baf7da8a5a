"""The allocation-free GEMM entry point, checked against the workspace-taking one.

apex_w4a4_gemm_noalloc serves callers that cannot allocate device memory while they run
(runtimes that budget every device byte in advance, plugin hosts whose allocator is off
limits, latency-critical paths that must avoid cudaMalloc/cudaFree stalls).  Its split-K
scratch is a fixed array inside the library, shared by every call on a device, so two
calls in a row also check that the second one does not see the first one's leftovers.

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


@pytest.mark.parametrize("M,N,K,gw", [(16, 2048, 8192, 128), (32, 1024, 4096, 512),
                                      (16, 256, 512, 128)])
def test_noalloc_matches_workspace_gemm_twice(apex, M, N, K, gw):
    a = synth.activations(M, K, "normal", 70 + M)
    w = synth.weights(N, K, 70 + N)
    a_d = torch.from_numpy(a).cuda()
    w_d = torch.from_numpy(w).cuda()
    ap, sa = apex.quantize_act(a_d, 128)
    wp, sw = apex.pack_weights(w_d, gw)
    ws = apex.workspace(M, N, K, 128, gw)
    y_ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm(M, N, K, 128, gw, ap, sa, wp, sw, y_ref, ws)
    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        apex.apex_w4a4_gemm_noalloc(M, N, K, 128, gw, ap, sa, wp, sw, y)
        outs.append(y)
    torch.cuda.synchronize()
    assert apex.apex_get_device_status() == 0
    ref = y_ref.cpu().numpy().astype(np.float64)
    for y in outs:
        got = y.cpu().numpy().astype(np.float64)
        ok, ratio = oracle.within_tolerance(got, ref)
        assert ok, f"no-alloc output differs from apex_w4a4_gemm (worst err/bound {ratio:.3f})"


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
