"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (the method: "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
Rebalancing", abstract -- W4A4 with per-128-group scales, INT4 products dequantised per
group):
  * packed int4 operands and fp16 scales: bit-exact;
  * per-group integer partials: bit-exact;
  * fp16 output: |y - y_ref| <= 2^-10 |y_ref| + 1e-3 max|y_ref| against the fp64 oracle.
Inputs are the seeded synthetic workloads of group_quantized_w4a4_b200.synth.
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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def f16(t):
    return host(t).view(np.uint16)


def check_status(apex):
    assert apex.apex_get_device_status() == 0


# ------------------------------------------------------------------ quantizer


@pytest.mark.parametrize("rows,K,dist", [(16, 512, "normal"), (37, 1024, "outlier"),
                                         (129, 2048, "student_t"), (1, 128, "normal")])
def test_quantize_act_bit_exact(apex, rows, K, dist):
    x = synth.activations(rows, K, dist, 7 + rows)
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    ap, sa = apex.quantize_act(dev(x), 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(ap), ap_ref)
    assert np.array_equal(f16(sa), sa_ref.view(np.uint16))
    check_status(apex)


@pytest.mark.parametrize("group", [128, 256, 512, 1024, 3072])
def test_pack_weights_bit_exact(apex, group):
    K = 3072
    w = synth.weights(70, K, 11)
    wp_ref, sw_ref = oracle.quantize_pack(w, group)
    wp, sw = apex.pack_weights(dev(w), group)
    torch.cuda.synchronize()
    assert np.array_equal(host(wp), wp_ref)
    assert np.array_equal(f16(sw), sw_ref.view(np.uint16))


def test_quantize_edge_values(apex):
    rng = np.random.default_rng(5)
    K = 512
    x = np.zeros((6, K), dtype=np.float16)
    x[1, :128] = 7.0
    x[1, 1:14] = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 4.5, 5.5, 6.5, -6.5, 0.25, 0.75]
    x[2] = (rng.integers(-7, 8, K) * 0.5).astype(np.float16)          # many ties
    x[3] = (rng.standard_normal(K) * 1e-5).astype(np.float16)         # subnormal scales
    x[4, 128:256] = np.float16(2.0 ** -24)                              # scale underflows
    x[5] = (rng.standard_normal(K) * 3000).astype(np.float16)          # large values
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    ap, sa = apex.quantize_act(dev(x), 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(ap), ap_ref)
    assert np.array_equal(f16(sa), sa_ref.view(np.uint16))


def test_quantize_full_size_bit_exact(apex):
    g = synth.workloads()["prefill_m4096_n8192_k8192"]
    x = synth.activations(g.M, g.K, g.act, g.seed)
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    ap, sa = apex.quantize_act(dev(x), 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(ap), ap_ref)
    assert np.array_equal(f16(sa), sa_ref.view(np.uint16))


# ------------------------------------------------------------------ integer partials


@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (1, 128, 128), (17, 200, 384),
                                   (64, 128, 256), (100, 384, 640), (129, 130, 256),
                                   (256, 256, 1024)])
def test_group_partials_bit_exact_random_bytes(apex, M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    ap = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)   # includes -8 nibbles
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    ref = oracle.group_partials(ap, wp, M, N, K, 128, 128)
    out = torch.empty((K // 128, M, N), dtype=torch.int32, device="cuda")
    apex.apex_w4a4_group_partials(M, N, K, dev(ap), dev(wp), out)
    torch.cuda.synchronize()
    assert np.array_equal(host(out).astype(np.int64), ref)
    check_status(apex)


def test_group_partials_extremes(apex):
    M, N, K = 16, 128, 256
    ap = np.full((M, K // 2), 0x88, dtype=np.uint8)                     # all -8
    wp = np.full((N, K // 2), 0x88, dtype=np.uint8)
    wp[1::2] = 0x77                                                     # all +7
    ref = oracle.group_partials(ap, wp, M, N, K, 128, 128)
    out = torch.empty((K // 128, M, N), dtype=torch.int32, device="cuda")
    apex.apex_w4a4_group_partials(M, N, K, dev(ap), dev(wp), out)
    torch.cuda.synchronize()
    assert np.array_equal(host(out).astype(np.int64), ref)
    assert ref.max() == 128 * 64 and ref.min() == -128 * 56


def test_group_partials_quantized_workload(apex):
    g = synth.workloads()["tiny_m16_n256_k512"]
    a, w = synth.make(g)
    ap, _ = oracle.quantize_pack(a, 128)
    wp, _ = oracle.quantize_pack(w, 128)
    ref = oracle.group_partials(ap, wp, g.M, g.N, g.K, 128, 128)
    out = torch.empty((g.K // 128, g.M, g.N), dtype=torch.int32, device="cuda")
    apex.apex_w4a4_group_partials(g.M, g.N, g.K, dev(ap), dev(wp), out)
    torch.cuda.synchronize()
    assert np.array_equal(host(out).astype(np.int64), ref)


def partials(apex, ap, wp, M, N, K, split):
    out = torch.full((K // 128, M, N), -1, dtype=torch.int32, device="cuda")
    apex.apex_debug_partials_split(split)
    apex.apex_w4a4_group_partials(M, N, K, ap, wp, out)
    torch.cuda.synchronize()
    check_status(apex)
    return host(out).astype(np.int64)


@pytest.mark.parametrize("split", [False, True])
def test_group_partials_full_decode_size(apex, split):
    """Every per-group partial of the headline decode shape (16 x 8192 x 8192, all 64 K-groups,
    every K coordinate and swizzle phase), bit-exact, on the GPU-quantized operands, whose
    packing is itself checked against the oracle; with split=True the work is divided as the
    bench's GEMM divides it (each tile over a 2-CTA cluster on a B200)."""
    g = synth.workloads()["decode_m16_n8192_k8192"]
    a, w = synth.make(g)
    ap, _ = apex.quantize_act(dev(a), 128)
    wp, _ = apex.pack_weights(dev(w), 128)
    torch.cuda.synchronize()
    ap_ref, _ = oracle.quantize_pack(a, 128)
    wp_ref, _ = oracle.quantize_pack(w, 128)
    assert np.array_equal(host(ap), ap_ref) and np.array_equal(host(wp), wp_ref)
    ref = oracle.group_partials(ap_ref, wp_ref, g.M, g.N, g.K, 128, 128)
    assert np.array_equal(partials(apex, ap, wp, g.M, g.N, g.K, split), ref)


# Split plans on a 148-SM B200: 2-, 3- and 4-way cluster splits, a 9-way split through
# global memory, true stream-K (CTAs holding pieces of two tiles) with 16-, 64- and
# 128-token tiles, and ragged M and N.
@pytest.mark.parametrize("M,N,K", [(16, 9472, 1024), (16, 6272, 1536), (5, 4736, 2048),
                                   (16, 2048, 8192), (16, 12800, 1024), (64, 6400, 1024),
                                   (200, 6400, 1024), (33, 1000, 2560)])
def test_group_partials_split_plans_bit_exact(apex, M, N, K):
    rng = np.random.default_rng(M + 3 * N + K)
    ap = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)   # includes -8 nibbles
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    ref = oracle.group_partials(ap, wp, M, N, K, 128, 128)
    assert np.array_equal(partials(apex, dev(ap), dev(wp), M, N, K, True), ref)


# ------------------------------------------------------------------ GEMM output


def run_gemm(apex, ap, sa, wp, sw, M, N, K, gw, ws=True):
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    w = apex.workspace(M, N, K, 128, gw) if ws else None
    apex.apex_w4a4_gemm(M, N, K, 128, gw, dev(ap), dev(sa), dev(wp), dev(sw), y, w)
    torch.cuda.synchronize()
    check_status(apex)
    return host(y).astype(np.float64)


def assert_close(y, ref, max_abs_ref=None):
    ok, ratio = oracle.within_tolerance(y, ref, max_abs_ref)
    assert ok, f"tolerance exceeded: worst err/bound = {ratio:.3f}"


@pytest.mark.parametrize("M,N,K,gw", [
    (16, 256, 512, 128), (1, 128, 128, 128), (15, 200, 384, 128), (17, 300, 1024, 512),
    (33, 128, 512, 512), (64, 256, 1024, 1024), (65, 129, 640, 128), (129, 257, 768, 768),
    (200, 384, 2048, 128), (256, 128, 1024, 256)])
def test_gemm_matches_oracle(apex, M, N, K, gw):
    a = synth.activations(M, K, "outlier", M + K)
    w = synth.weights(N, K, N + K)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, gw)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, gw)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, gw), ref)


def test_gemm_without_workspace_matches(apex):
    M, N, K = 16, 1024, 4096
    a = synth.activations(M, K, "normal", 3)
    w = synth.weights(N, K, 3)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, 128, ws=False), ref)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, 128, ws=True), ref)


def test_gemm_random_bytes_and_scales(apex):
    rng = np.random.default_rng(99)
    M, N, K = 48, 256, 1024
    ap = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    wp = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.uniform(0.01, 4.0, size=(M, K // 128)).astype(np.float16)
    sw = rng.uniform(1e-4, 0.05, size=(N, K // 128)).astype(np.float16)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, 128), ref)


def test_gemm_split_k_is_deterministic(apex):
    M, N, K = 16, 2048, 8192
    a = synth.activations(M, K, "normal", 1)
    w = synth.weights(N, K, 1)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    ws = apex.workspace(M, N, K)
    assert ws is not None
    args = [dev(x) for x in (ap, sa, wp, sw)]
    outs = []
    for _ in range(3):
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        apex.apex_w4a4_gemm(M, N, K, 128, 128, *args, y, ws)
        outs.append(y)
    torch.cuda.synchronize()
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    assert int(ws[:256].sum()) == 0        # arrival counters are left at zero


@pytest.mark.parametrize("M,ways", [(16, 2), (16, 3), (16, 4), (32, 2), (5, 4)])
def test_gemm_split_over_a_cluster_matches_oracle(apex, M, ways):
    # N chosen so that every tile is split `ways` ways on this device (one CTA per SM):
    # 16- and 32-token tiles split 2-4 ways run as thread-block clusters; a pair exchanges
    # halves of its sums and each CTA writes half of the tile's tokens, larger clusters add
    # the parts in the owner's shared memory.  The last tile is ragged.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    N = 128 * (sms // ways) - 50
    K = 128 * 4 * ways * 2             # two pipeline stages per CTA
    a = synth.activations(M, K, "outlier", 40 + ways)
    w = synth.weights(N, K, 40 + ways)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    y = run_gemm(apex, ap, sa, wp, sw, M, N, K, 128)
    assert_close(y, ref)
    assert np.array_equal(y, run_gemm(apex, ap, sa, wp, sw, M, N, K, 128))   # deterministic


def test_gemm_scale_linearity(apex):
    M, N, K = 32, 256, 1024
    a = synth.activations(M, K, "normal", 8)
    w = synth.weights(N, K, 8)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    y0 = run_gemm(apex, ap, sa, wp, sw, M, N, K, 128)
    sw2 = sw.copy()
    sw2[5] = (sw2[5].astype(np.float32) * 2).astype(np.float16)
    y1 = run_gemm(apex, ap, sa, wp, sw2, M, N, K, 128)
    want = y0.copy()
    want[:, 5] *= 2
    assert np.array_equal(y1, want)


@pytest.mark.parametrize("name", ["tiny_m16_n256_k512", "decode_m16_n8192_k8192"])
def test_gemm_full_workloads(apex, name):
    g = synth.workloads()[name]
    a, w = synth.make(g)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, g.gw)
    ref = oracle.gemm(ap, sa, wp, sw, g.M, g.N, g.K, 128, g.gw)
    assert_close(run_gemm(apex, ap, sa, wp, sw, g.M, g.N, g.K, g.gw), ref)


SAMPLED = ["prefill_m4096_n8192_k8192", "mlp_up_m2048_n28672_k8192",
           "mlp_down_m2048_n8192_k28672", "sweep_m1_gw128", "sweep_m128_gw512",
           "sweep_m1024_gw8192", "sweep_m4096_gw512", "sweep_m16_gw8192"]


@pytest.mark.parametrize("name", SAMPLED)
def test_gemm_large_workloads_sampled_rows(apex, name):
    """Full-size problem in the benchmark's launch configuration; the whole pipeline
    (quantizer + GEMM) runs on the GPU, the oracle checks sampled output rows."""
    g = synth.workloads()[name]
    a, w = synth.make(g)
    a_d, w_d = dev(a), dev(w)
    ap, sa = apex.quantize_act(a_d, 128)
    wp, sw = apex.pack_weights(w_d, g.gw)
    ws = apex.workspace(g.M, g.N, g.K, 128, g.gw)
    y = apex.gemm(ap, sa, wp, sw, 128, g.gw, ws=ws)
    torch.cuda.synchronize()
    check_status(apex)
    rng = np.random.default_rng(0)
    cand = {0, g.M - 1, min(127, g.M - 1), min(128, g.M - 1), g.M // 2}
    cand |= set(rng.integers(0, g.M, size=min(g.M, 12)).tolist())
    rows = np.array(sorted(cand), dtype=np.int64)
    ap_h, sa_h, wp_h, sw_h = host(ap), host(sa), host(wp), host(sw)
    # the GPU-packed operands are themselves checked against the oracle's quantizer, whole,
    # before any of them serves as oracle input
    ap_ref, sa_ref = oracle.quantize_pack(a, 128)
    assert np.array_equal(ap_h, ap_ref)
    assert np.array_equal(sa_h.view(np.uint16), sa_ref.view(np.uint16))
    wp_ref, sw_ref = oracle.quantize_pack(w, g.gw)
    assert np.array_equal(wp_h, wp_ref)
    assert np.array_equal(sw_h.view(np.uint16), sw_ref.view(np.uint16))
    ref = oracle.gemm(ap_ref, sa_ref, wp_ref, sw_ref, g.M, g.N, g.K, 128, g.gw, rows=rows)
    got = host(y)[rows].astype(np.float64)
    # max|ref| over the whole output is at least the sampled max: using the sampled max
    # makes the absolute term of the bound no looser than the stated rule.
    assert_close(got, ref)


# ------------------------------------------------------------------ expanded activations


def expected_expanded(q):
    """16*q in the GEMM operand order: per 8 elements, k0,k2,k4,k6 then k1,k3,k5,k7."""
    rows, K = q.shape
    blk = q.reshape(rows, K // 8, 8)
    order = blk[:, :, [0, 2, 4, 6, 1, 3, 5, 7]] * 16
    return order.reshape(rows, K).astype(np.int8).view(np.uint8)


@pytest.mark.parametrize("rows,K,dist", [(16, 512, "normal"), (130, 2048, "outlier"),
                                         (1, 128, "student_t")])
def test_quantize_expanded_bit_exact(apex, rows, K, dist):
    x = synth.activations(rows, K, dist, 17 + rows)
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    q8, sa = apex.quantize_act_expanded(dev(x), 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(q8), expected_expanded(oracle.unpack(ap_ref, K).astype(np.int64)))
    assert np.array_equal(f16(sa), sa_ref.view(np.uint16))


def run_gemm_expanded(apex, x, wp, sw, M, N, K, gw):
    q8, sa = apex.quantize_act_expanded(dev(x), 128)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    w = apex.workspace(M, N, K, 128, gw)
    apex.apex_w4a4_gemm_expanded(M, N, K, 128, gw, q8, sa, dev(wp), dev(sw), y, w)
    torch.cuda.synchronize()
    check_status(apex)
    return host(y).astype(np.float64)


@pytest.mark.parametrize("M,N,K,gw", [(16, 256, 512, 128), (130, 257, 1024, 128),
                                      (256, 384, 2048, 512), (200, 128, 768, 768),
                                      (129, 1024, 4096, 128)])
def test_gemm_expanded_matches_oracle(apex, M, N, K, gw):
    a = synth.activations(M, K, "outlier", 3 * M + K)
    w = synth.weights(N, K, N + 3 * K)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, gw)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, gw)
    assert_close(run_gemm_expanded(apex, a, wp, sw, M, N, K, gw), ref)


@pytest.mark.parametrize("name", ["prefill_m4096_n8192_k8192", "mlp_down_m2048_n8192_k28672",
                                  "sweep_m1024_gw512"])
def test_gemm_expanded_large_sampled_rows(apex, name):
    g = synth.workloads()[name]
    a, w = synth.make(g)
    wp, sw = apex.pack_weights(dev(w), g.gw)
    q8, sa = apex.quantize_act_expanded(dev(a), 128)
    y = torch.empty((g.M, g.N), dtype=torch.float16, device="cuda")
    ws = apex.workspace(g.M, g.N, g.K, 128, g.gw)
    apex.apex_w4a4_gemm_expanded(g.M, g.N, g.K, 128, g.gw, q8, sa, wp, sw, y, ws)
    torch.cuda.synchronize()
    check_status(apex)
    rows = np.array(sorted({0, 1, 127, 128, g.M // 3, g.M - 1}), dtype=np.int64)
    ap_ref, sa_ref = oracle.quantize_pack(a[rows], 128)
    ref = oracle.gemm(ap_ref, sa_ref, host(wp), host(sw), rows.size, g.N, g.K, 128, g.gw)
    assert_close(host(y)[rows].astype(np.float64), ref)


# ------------------------------------------------------------------ quantize + GEMM in one call


def run_linear(apex, x, wp, sw, M, N, K, gw):
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    w = apex.workspace(M, N, K, 128, gw, linear=True)
    apex.apex_w4a4_linear(M, N, K, 128, gw, dev(x), dev(wp), dev(sw), y, w)
    torch.cuda.synchronize()
    check_status(apex)
    return y


@pytest.mark.parametrize("M,N,K,gw", [(1, 256, 512, 128), (5, 384, 1024, 128),
                                      (16, 256, 512, 128), (16, 1024, 2048, 512),
                                      (17, 300, 1024, 128), (32, 512, 4096, 128),
                                      (48, 256, 1024, 1024), (64, 640, 2048, 128),
                                      (65, 256, 768, 128), (200, 384, 1024, 256)])
def test_linear_matches_oracle_and_two_step_path(apex, M, N, K, gw):
    """apex_w4a4_linear (quantize into its workspace, then the GEMM): within tolerance of the
    oracle and bit-identical to the separate quantize and GEMM calls."""
    a = synth.activations(M, K, "outlier", 5 * M + K)
    w = synth.weights(N, K, 5 * N + K)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, gw)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, gw)
    y = run_linear(apex, a, wp, sw, M, N, K, gw)
    assert_close(host(y).astype(np.float64), ref)
    if M >= 128:
        q8, sa2 = apex.quantize_act_expanded(dev(a), 128)
        y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
        apex.apex_w4a4_gemm_expanded(M, N, K, 128, gw, q8, sa2, dev(wp), dev(sw), y2,
                                     apex.workspace(M, N, K, 128, gw))
    else:
        ap2, sa2 = apex.quantize_act(dev(a), 128)
        y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")
        apex.apex_w4a4_gemm(M, N, K, 128, gw, ap2, sa2, dev(wp), dev(sw), y2,
                            apex.workspace(M, N, K, 128, gw))
    torch.cuda.synchronize()
    check_status(apex)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_linear_decode_workload_and_edge_values(apex):
    """The decode workload end to end, and a batch with all-zero, tiny and tie-valued rows."""
    g = synth.workloads()["decode_m16_n8192_k8192"]
    a, w = synth.make(g)
    a[3] = 0.0                                   # all-zero rows: scale 0, q = 0
    a[4, :] = np.float16(1e-7)                   # scale underflows to fp16 zero
    a[5, :128] = np.float16(7.0)                 # s = 1 exactly, then ties
    a[5, 0:8] = np.array([0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, -3.5], dtype=np.float16)
    wp, sw = oracle.quantize_pack(w, g.gw)
    ap, sa = oracle.quantize_pack(a, 128)
    ref = oracle.gemm(ap, sa, wp, sw, g.M, g.N, g.K, 128, g.gw)
    y = run_linear(apex, a, wp, sw, g.M, g.N, g.K, g.gw)
    assert_close(host(y).astype(np.float64), ref)


def test_linear_refuses_a_missing_workspace(apex):
    M, N, K = 16, 256, 512
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    wp = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.zeros((N, K // 128), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_linear(M, N, K, 128, 128, x, wp, sw, y, None)
    assert e.value.code == apex.APEX_ERR_INVALID_ARG


# ------------------------------------------------------------------ failure path


def test_pipeline_wait_timeout_is_reported_and_context_survives(apex):
    M, N, K = 16, 256, 1024
    a = synth.activations(M, K, "normal", 2)
    w = synth.weights(N, K, 2)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    args = [dev(x) for x in (ap, sa, wp, sw)]
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    apex.apex_set_wait_limit_ns(50_000_000)           # 50 ms
    try:
        apex.apex_debug_withhold_step(1)              # one bulk copy never issued
        apex.apex_w4a4_gemm(M, N, K, 128, 128, *args, y, None)
        assert apex.apex_get_device_status() == apex.APEX_ERR_TIMEOUT
    finally:
        apex.apex_set_wait_limit_ns(2_000_000_000)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, 128), ref)


def test_cluster_wait_timeout_is_reported_and_context_survives(apex):
    # The same failure inside a clustered split: every CTA gives up at its second stage,
    # the partners still send their parts, the owners still take them, and the launch ends.
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M, N, K = 16, 128 * (sms // 2), 2048
    a = synth.activations(M, K, "normal", 5)
    w = synth.weights(N, K, 5)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    args = [dev(x) for x in (ap, sa, wp, sw)]
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    ws = apex.workspace(M, N, K)
    assert ws is not None
    apex.apex_set_wait_limit_ns(50_000_000)           # 50 ms
    try:
        apex.apex_debug_withhold_step(1)              # every CTA's second stage never issued
        apex.apex_w4a4_gemm(M, N, K, 128, 128, *args, y, ws)
        assert apex.apex_get_device_status() == apex.APEX_ERR_TIMEOUT
    finally:
        apex.apex_set_wait_limit_ns(2_000_000_000)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128)
    assert_close(run_gemm(apex, ap, sa, wp, sw, M, N, K, 128), ref)


# ------------------------------------------------------------------ quantized output


QUANT_OUT_SHAPES = [
    (16, 9472, 1024),    # 74 tiles: 2-CTA clusters on a B200
    (16, 1024, 1024),    # split through global memory
    (16, 256, 512),      # whole tiles
    (1, 384, 1024),
    (17, 2048, 1024),    # 32-token tiles, split through global memory
    (64, 1024, 512),
    (100, 512, 768),
    (200, 384, 1024),    # 128-token tiles, ragged token block
    (16, 12800, 1024),   # stream-K: 200 units over 148 CTAs, pieces of two tiles per CTA
    (200, 6400, 1024),   # stream-K with 128-token tiles
]


@pytest.mark.parametrize("M,N,K", QUANT_OUT_SHAPES)
@pytest.mark.parametrize("expanded_in", [False, True])
@pytest.mark.parametrize("expanded_out", [False, True])
def test_gemm_quantized_output_is_the_quantizer_of_y(apex, M, N, K, expanded_in, expanded_out):
    """The fused output equals the oracle's activation quantizer applied to the fp16 Y the
    same call wrote (bit-exact), and Y itself meets the GEMM bar."""
    x = synth.activations(M, K, "outlier", 90 + M)
    w = synth.weights(N, K, 90 + N)
    ap, sa = oracle.quantize_pack(x, 128)
    wp, sw = oracle.quantize_pack(w, 128)
    if expanded_in:
        a_q, a_s = apex.quantize_act_expanded(dev(x), 128)
        fn = apex.apex_w4a4_gemm_expanded_quant
    else:
        a_q, a_s = dev(ap), dev(sa)
        fn = apex.apex_w4a4_gemm_quant
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    yq = torch.empty((M, N if expanded_out else N // 2), dtype=torch.uint8, device="cuda")
    ys = torch.empty((M, N // 128), dtype=torch.float16, device="cuda")
    ws = apex.workspace(M, N, K)
    fn(M, N, K, 128, 128, a_q, a_s, dev(wp), dev(sw), y, yq, ys, expanded_out, ws)
    torch.cuda.synchronize()
    check_status(apex)
    y_h = host(y)
    assert_close(y_h.astype(np.float64), oracle.gemm(ap, sa, wp, sw, M, N, K, 128, 128))
    q_ref, s_ref = oracle.quantize_pack(y_h, 128)
    if expanded_out:
        assert np.array_equal(host(yq), expected_expanded(oracle.unpack(q_ref, N).astype(np.int64)))
    else:
        assert np.array_equal(host(yq), q_ref)
    assert np.array_equal(f16(ys), s_ref.view(np.uint16))
    # without Y: the same quantized output
    yq2, ys2 = torch.zeros_like(yq), torch.zeros_like(ys)
    fn(M, N, K, 128, 128, a_q, a_s, dev(wp), dev(sw), None, yq2, ys2, expanded_out, ws)
    torch.cuda.synchronize()
    check_status(apex)
    assert torch.equal(yq2, yq) and torch.equal(ys2, ys)


def test_gemm_quantized_output_argument_rules(apex):
    M, N, K = 16, 200, 256                 # N not a multiple of 128
    a = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    s = torch.zeros((M, K // 128), dtype=torch.float16, device="cuda")
    wq = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    wsc = torch.zeros((N, K // 128), dtype=torch.float16, device="cuda")
    yq = torch.zeros((M, N), dtype=torch.uint8, device="cuda")
    ys = torch.zeros((M, 2), dtype=torch.float16, device="cuda")
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_quant(M, N, K, 128, 128, a, s, wq, wsc, None, yq, ys)
    assert e.value.code == apex.APEX_ERR_UNSUPPORTED
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_quant(M, 256, K, 128, 128, a, s, wq, wsc, None, None, ys)
    assert e.value.code == apex.APEX_ERR_INVALID_ARG


def test_chained_layers_through_the_quantized_output(apex):
    """Two W4A4 layers, the first one's quantized output fed straight to the second: the
    second's result equals the oracle GEMM on the operands the first one produced."""
    M, K, H, N = 16, 1024, 2048, 512
    x = synth.activations(M, K, "normal", 123)
    w1, w2 = synth.weights(H, K, 124), synth.weights(N, H, 125)
    ap, sa = oracle.quantize_pack(x, 128)
    w1p, w1s = oracle.quantize_pack(w1, 128)
    w2p, w2s = oracle.quantize_pack(w2, 128)
    hq = torch.empty((M, H // 2), dtype=torch.uint8, device="cuda")
    hs = torch.empty((M, H // 128), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_quant(M, H, K, 128, 128, dev(ap), dev(sa), dev(w1p), dev(w1s), None,
                              hq, hs, False, apex.workspace(M, H, K))
    apex.apex_w4a4_gemm(M, N, H, 128, 128, hq, hs, dev(w2p), dev(w2s), y, apex.workspace(M, N, H))
    torch.cuda.synchronize()
    check_status(apex)
    ref = oracle.gemm(host(hq), host(hs), w2p, w2s, M, N, H, 128, 128)
    assert_close(host(y).astype(np.float64), ref)


@pytest.mark.parametrize("M", [2048, 16])
def test_gemm_quantized_output_full_size_sampled_rows(apex, M):
    """The up-projection of the MLP pair (8192 -> 28672) at full size, in the form the chained
    step times (expanded activations from M = 128 on): sampled rows of Y meet the GEMM bar,
    and the same rows of the quantized output, in both output forms, are the oracle's
    quantizer applied to Y, bit for bit."""
    K, N = 8192, 28672
    x = synth.activations(M, K, "student_t", 7)
    w = synth.weights(N, K, 8)
    wp, sw = apex.pack_weights(dev(w), 128)
    expanded_in = M >= 128
    if expanded_in:
        a_q, a_s = apex.quantize_act_expanded(dev(x), 128)
        fn = apex.apex_w4a4_gemm_expanded_quant
    else:
        a_q, a_s = apex.quantize_act(dev(x), 128)
        fn = apex.apex_w4a4_gemm_quant
    ws = apex.workspace(M, N, K)
    rows = np.array(sorted({r for r in (0, 1, 127, 128, M // 3, M - 1) if r < M}), dtype=np.int64)
    ap_ref, sa_ref = oracle.quantize_pack(x[rows], 128)
    ref = oracle.gemm(ap_ref, sa_ref, host(wp), host(sw), rows.size, N, K, 128, 128)
    for expanded_out in (False, True):
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        yq = torch.empty((M, N if expanded_out else N // 2), dtype=torch.uint8, device="cuda")
        ys = torch.empty((M, N // 128), dtype=torch.float16, device="cuda")
        fn(M, N, K, 128, 128, a_q, a_s, wp, sw, y, yq, ys, expanded_out, ws)
        torch.cuda.synchronize()
        check_status(apex)
        y_rows = host(y)[rows]
        assert_close(y_rows.astype(np.float64), ref)
        q_ref, s_ref = oracle.quantize_pack(y_rows, 128)
        if expanded_out:
            want = expected_expanded(oracle.unpack(q_ref, N).astype(np.int64))
        else:
            want = q_ref
        assert np.array_equal(host(yq)[rows], want)
        assert np.array_equal(f16(ys)[rows], s_ref.view(np.uint16))
