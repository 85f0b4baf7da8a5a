"""GPU parity of the E4M3-carrier path (many-token GEMMs) against the CPU oracle.

The path carries the same 4-bit values q as E4M3 codes, one byte per element, so that the
tensor cores' fp32-accumulating kind::f8f6f4 MMA returns every K-group's integer partial
directly ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing",
abstract: INT4 products, per-group dequantisation).  Bars:
  * codes: the E4M3 encoding of the oracle's q, bit for bit (the encoding itself is taken
    from torch's float8_e4m3fn conversion, a library routine independent of this code);
    scales bit-exact;
  * per-group partials: bit-exact against the oracle's int64 partials, including the
    extreme sums (+-8192) and odd sums near them, where an inexact fp32 accumulation
    would show;
  * fp16 output: the oracle bound |y - y_ref| <= 2^-10 |y_ref| + 1e-3 max|y_ref|, and
    bit-identical to the int8 path's whole-tile GEMM, which forms the same fp32 products
    and adds the groups in the same order.
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


def e4m3_codes(q):
    """E4M3 bytes of integer values (torch's float8_e4m3fn conversion)."""
    t = torch.from_numpy(np.asarray(q, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def check_status(apex):
    assert apex.apex_get_device_status() == 0


def assert_close(y, ref):
    ok, ratio = oracle.within_tolerance(y, ref)
    assert ok, f"tolerance exceeded: worst err/bound = {ratio:.3f}"


# ------------------------------------------------------------------ codes


@pytest.mark.parametrize("rows,K,dist", [(16, 512, "normal"), (130, 2048, "outlier"),
                                         (1, 128, "student_t"), (257, 1024, "normal")])
def test_quantize_act_fp8_codes(apex, rows, K, dist):
    x = synth.activations(rows, K, dist, 300 + rows)
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    codes, sa = apex.quantize_act_fp8(dev(x), 128)
    torch.cuda.synchronize()
    assert np.array_equal(host(codes), e4m3_codes(oracle.unpack(ap_ref, K)))
    assert np.array_equal(host(sa).view(np.uint16), sa_ref.view(np.uint16))


@pytest.mark.parametrize("group", [128, 512, 3072])
def test_pack_weights_fp8_codes(apex, group):
    K = 3072
    w = synth.weights(70, K, 13)
    wp_ref, sw_ref = oracle.quantize_pack(w, group)
    codes, sw = apex.pack_weights_fp8(dev(w), group)
    torch.cuda.synchronize()
    assert np.array_equal(host(codes), e4m3_codes(oracle.unpack(wp_ref, K)))
    assert np.array_equal(host(sw).view(np.uint16), sw_ref.view(np.uint16))


def test_unpack_int4_fp8_every_byte(apex):
    rng = np.random.default_rng(4)
    packed = np.tile(np.arange(256, dtype=np.uint8), (3, 8))           # every byte value
    packed = np.concatenate([packed, rng.integers(0, 256, (5, 2048), dtype=np.uint8)])
    rows, K = packed.shape[0], packed.shape[1] * 2
    codes = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    apex.apex_unpack_int4_fp8(dev(packed), rows, K, codes)
    torch.cuda.synchronize()
    assert np.array_equal(host(codes), e4m3_codes(oracle.unpack(packed, K)))


# ------------------------------------------------------------------ partials


def partials_fp8(apex, qa, qw):
    M, K = qa.shape
    N = qw.shape[0]
    out = torch.full((K // 128, M, N), -1, dtype=torch.int32, device="cuda")
    apex.apex_w4a4_group_partials_fp8(M, N, K, dev(e4m3_codes(qa)), dev(e4m3_codes(qw)), out)
    torch.cuda.synchronize()
    check_status(apex)
    return host(out).astype(np.int64)


def pack(q):
    q = np.asarray(q, dtype=np.int64)
    lo, hi = q[:, 0::2] & 0xF, q[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


@pytest.mark.parametrize("M,N,K", [(16, 256, 512), (1, 128, 128), (129, 300, 640),
                                   (128, 256, 1024), (200, 520, 256), (300, 1000, 1152)])
def test_group_partials_fp8_random_values(apex, M, N, K):
    rng = np.random.default_rng(M + N + K)
    qa = rng.integers(-8, 8, size=(M, K))
    qw = rng.integers(-8, 8, size=(N, K))
    ref = oracle.group_partials(pack(qa), pack(qw), M, N, K, 128, 128)
    assert np.array_equal(partials_fp8(apex, qa, qw), ref)


def test_group_partials_fp8_extreme_and_odd_sums(apex):
    """Sums at and next to the largest magnitudes a group can reach: 128 * (-8)(-8) = 8192,
    128 * 7 * (-8) = -7168, and 127 products of 64 plus one product of two odd values
    (8128 + 49 = 8177, 8128 - 7, ...), the odd position moving from group to group, so that
    a lost low bit anywhere in the accumulation shows."""
    M, N, K = 128, 256, 512
    G = K // 128
    rng = np.random.default_rng(1)
    pos = [g * 128 + int(rng.integers(0, 128)) for g in range(G)]
    qa = np.full((M, K), -8, dtype=np.int64)
    qw = np.full((N, K), -8, dtype=np.int64)
    qw[1::4] = 7
    for r in range(1, M, 3):
        for p in pos:
            qa[r, p] = rng.choice([7, -7, 5, 1])
    for r in range(2, N, 4):
        for p in pos:
            qw[r, p] = rng.choice([7, -1, 3, -5])
    ref = oracle.group_partials(pack(qa), pack(qw), M, N, K, 128, 128)
    assert ref.max() == 8192 and ref.min() == -7168
    odd = ref[:, 1::3, 2::4]
    assert np.all(odd % 2 == 1) and odd.max() == 8177
    assert np.array_equal(partials_fp8(apex, qa, qw), ref)


# ------------------------------------------------------------------ GEMM


def run_fp8(apex, a, w, M, N, K, gw):
    ac, sa = apex.quantize_act_fp8(dev(a), 128)
    wc, sw = apex.pack_weights_fp8(dev(w), gw)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8(M, N, K, 128, gw, ac, sa, wc, sw, y)
    torch.cuda.synchronize()
    check_status(apex)
    return y


@pytest.mark.parametrize("M,N,K,gw", [
    (16, 256, 512, 128), (1, 128, 128, 128), (129, 300, 640, 128), (128, 256, 1024, 512),
    (200, 520, 1024, 1024), (256, 512, 2048, 128), (300, 1000, 1152, 384),
    (1100, 2100, 1024, 128), (64, 8192, 1024, 128)])
def test_gemm_fp8_matches_oracle(apex, M, N, K, gw):
    a = synth.activations(M, K, "outlier", 2 * M + K)
    w = synth.weights(N, K, 2 * N + K)
    ap, sa = oracle.quantize_pack(a, 128)
    wp, sw = oracle.quantize_pack(w, gw)
    ref = oracle.gemm(ap, sa, wp, sw, M, N, K, 128, gw)
    assert_close(host(run_fp8(apex, a, w, M, N, K, gw)).astype(np.float64), ref)


def test_gemm_fp8_from_unpacked_weights(apex):
    """Weights packed as int4 and turned into codes with apex_unpack_int4_fp8 give the same
    output as codes quantized straight from fp16."""
    M, N, K = 200, 512, 1024
    a = synth.activations(M, K, "normal", 5)
    w = synth.weights(N, K, 5)
    y0 = run_fp8(apex, a, w, M, N, K, 128)
    wp, sw = apex.pack_weights(dev(w), 128)
    wc = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    apex.apex_unpack_int4_fp8(wp, N, K, wc)
    ac, sa = apex.quantize_act_fp8(dev(a), 128)
    y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8(M, N, K, 128, 128, ac, sa, wc, sw, y1)
    torch.cuda.synchronize()
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))


FULL = ["prefill_m4096_n8192_k8192", "mlp_up_m2048_n28672_k8192", "mlp_down_m2048_n8192_k28672",
        "sweep_m1024_gw128", "sweep_m4096_gw512", "sweep_m4096_gw8192", "sweep_m128_gw128"]


@pytest.mark.parametrize("name", FULL)
def test_gemm_fp8_full_size_sampled_rows(apex, name):
    """The full workload in the benchmark's launch configuration: codes and scales checked
    whole against the oracle's quantizer, sampled rows of Y against the oracle GEMM, and --
    where the int8 path runs whole tiles with the same group order -- the whole Y bit for bit
    against apex_w4a4_gemm_expanded."""
    g = synth.workloads()[name]
    a, w = synth.make(g)
    ac, sa = apex.quantize_act_fp8(dev(a), 128)
    wc, sw = apex.pack_weights_fp8(dev(w), g.gw)
    y = torch.empty((g.M, g.N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8(g.M, g.N, g.K, 128, g.gw, ac, sa, wc, sw, y)
    torch.cuda.synchronize()
    check_status(apex)
    ap_ref, sa_ref = oracle.quantize_pack(a, 128)
    wp_ref, sw_ref = oracle.quantize_pack(w, g.gw)
    assert np.array_equal(host(sa).view(np.uint16), sa_ref.view(np.uint16))
    assert np.array_equal(host(sw).view(np.uint16), sw_ref.view(np.uint16))
    assert np.array_equal(host(ac), e4m3_codes(oracle.unpack(ap_ref, g.K)))
    assert np.array_equal(host(wc), e4m3_codes(oracle.unpack(wp_ref, g.K)))
    rng = np.random.default_rng(3)
    cand = {0, 1, 127, 128, g.M // 3, g.M - 1} | set(rng.integers(0, g.M, 8).tolist())
    rows = np.array(sorted(r for r in cand if r < g.M), dtype=np.int64)
    ref = oracle.gemm(ap_ref, sa_ref, wp_ref, sw_ref, g.M, g.N, g.K, 128, g.gw, rows=rows)
    assert_close(host(y)[rows].astype(np.float64), ref)
    plan = apex.apex_debug_gemm_plan(g.M, g.N, g.K, torch.cuda.get_device_properties(0)
                                     .multi_processor_count)
    if g.gw != g.K and plan["bt"] == 128 and not plan["split_k"]:
        q8, sa8 = apex.quantize_act_expanded(dev(a), 128)
        wp, sw2 = apex.pack_weights(dev(w), g.gw)
        y8 = torch.empty_like(y)
        apex.apex_w4a4_gemm_expanded(g.M, g.N, g.K, 128, g.gw, q8, sa8, wp, sw2, y8,
                                     apex.workspace(g.M, g.N, g.K, 128, g.gw))
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y8.view(torch.int16))


def test_gemm_fp8_argument_errors(apex):
    t = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    h = torch.zeros(64, dtype=torch.float16, device="cuda")
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_fp8(16, 128, 200, 128, 128, t, h, t, h, h)   # K % 128
    assert e.value.code == apex.APEX_ERR_INVALID_ARG
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_fp8(16, 128, 256, 64, 128, t, h, t, h, h)    # group_a != 128
    assert e.value.code == apex.APEX_ERR_UNSUPPORTED
    with pytest.raises(apex.ApexError) as e:
        apex.apex_w4a4_gemm_fp8(16, 128, 256, 128, 128, t[1:], h, t, h, h)   # misaligned
    assert e.value.code == apex.APEX_ERR_ALIGNMENT


# ------------------------------------------------------------------ outlier dual path


def dual_inputs(apex, x, w, ch, Cp, gw=128):
    """Device operands of the dual path: the outlier list, the gathered weight columns, the
    weight codes, and the dual quantizer's outputs (E4M3 codes, scales, x_out)."""
    M, K = x.shape
    N = w.shape[0]
    ch_d = dev(np.ascontiguousarray(ch, dtype=np.int32))
    w_d = dev(w)
    w_out = torch.full((N, Cp), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_gather_weight_columns(w_d, N, K, ch_d, len(ch), w_out, Cp)
    wc, sw = apex.pack_weights_fp8(w_d, gw)
    q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M, K // 128), dtype=torch.float16, device="cuda")
    x_out = torch.full((M, Cp), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_quantize_act_int4_dual(dev(x), M, K, 128, ch_d, len(ch), apex.APEX_FORM_FP8, q, s,
                                     x_out, Cp)
    return q, s, x_out, wc, sw, w_out


@pytest.mark.parametrize("M,K,C,Cp", [(16, 1024, 11, 64), (37, 2048, 21, 64), (3, 256, 1, 64),
                                      (130, 4096, 82, 128)])
@pytest.mark.parametrize("form", [0, 1, 2])
def test_quantize_dual_is_the_oracle_split_then_quantizer(apex, M, K, C, Cp, form):
    x = synth.activations(M, K, "outlier", 70 + M)
    ch = np.sort(np.random.default_rng(K + C).choice(K, size=C, replace=False))
    ch_d = dev(ch.astype(np.int32))
    q = torch.empty((M, K // 2 if form == 0 else K), dtype=torch.uint8, device="cuda")
    s = torch.empty((M, K // 128), dtype=torch.float16, device="cuda")
    x_out = torch.full((M, Cp), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_quantize_act_int4_dual(dev(x), M, K, 128, ch_d, C, form, q, s, x_out, Cp)
    torch.cuda.synchronize()
    x_in, x_out_ref = oracle.split_outlier_channels(x, ch)
    ap_ref, sa_ref = oracle.quantize_pack(x_in, 128)
    qv = oracle.unpack(ap_ref, K).astype(np.int64)
    if form == 0:
        assert np.array_equal(host(q), ap_ref)
    elif form == 1:
        blk = qv.reshape(M, K // 8, 8)[:, :, [0, 2, 4, 6, 1, 3, 5, 7]] * 16
        assert np.array_equal(host(q), blk.reshape(M, K).astype(np.int8).view(np.uint8))
    else:
        assert np.array_equal(host(q), e4m3_codes(qv))
    assert np.array_equal(host(s).view(np.uint16), sa_ref.view(np.uint16))
    xo = host(x_out).view(np.uint16)
    assert np.array_equal(xo[:, :C], x_out_ref.view(np.uint16))
    assert not np.any(xo[:, C:])


def test_gather_weight_columns_exact(apex):
    N, K = 300, 1024
    w = synth.weights(N, K, 71)
    ch = synth.outlier_channels(K, 72)
    ch_d = dev(ch.astype(np.int32))
    w_out = torch.full((N, 64), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_gather_weight_columns(dev(w), N, K, ch_d, len(ch), w_out, 64)
    torch.cuda.synchronize()
    got = host(w_out).view(np.uint16)
    assert np.array_equal(got[:, :len(ch)], np.ascontiguousarray(w[:, ch]).view(np.uint16))
    assert not np.any(got[:, len(ch):])


@pytest.mark.parametrize("M,N,K,C,gw", [(16, 256, 512, 5, 128), (1, 384, 1024, 11, 128),
                                        (129, 300, 1024, 82, 128), (200, 640, 2048, 21, 512),
                                        (256, 512, 2048, 64, 2048), (300, 1000, 1152, 130, 128)])
def test_gemm_fp8_dual_matches_oracle(apex, M, N, K, C, gw):
    x = synth.activations(M, K, "outlier", 80 + M)
    w = synth.weights(N, K, 80 + N)
    ch = np.sort(np.random.default_rng(M + C).choice(K, size=C, replace=False))
    Cp = -(-C // 64) * 64
    q, s, x_out, wc, sw, w_out = dual_inputs(apex, x, w, ch, Cp, gw)
    y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8_dual(M, N, K, 128, gw, q, s, wc, sw, x_out, w_out, Cp, y)
    torch.cuda.synchronize()
    check_status(apex)
    x_in, x_out_ref = oracle.split_outlier_channels(x, ch)
    ap, sa = oracle.quantize_pack(x_in, 128)
    wp, swr = oracle.quantize_pack(w, gw)
    ref = oracle.gemm_dual(ap, sa, wp, swr, x_out_ref, np.ascontiguousarray(w[:, ch]), M, N, K,
                           128, gw)
    assert_close(host(y).astype(np.float64), ref)


def test_gemm_fp8_dual_full_size_prefill(apex):
    """The prefill workload with its own outlier channels (1% of K, x20) through the dual
    path; sampled rows against the oracle, and the dual path's error against the exact fp16
    product below the plain W4A4 path's."""
    g = synth.workloads()["prefill_m4096_n8192_k8192"]
    a, w = synth.make(g)
    ch = synth.outlier_channels(g.K, g.seed * 16 + 2)
    C = len(ch)
    Cp = -(-C // 64) * 64
    q, s, x_out, wc, sw, w_out = dual_inputs(apex, a, w, ch, Cp)
    y = torch.empty((g.M, g.N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8_dual(g.M, g.N, g.K, 128, 128, q, s, wc, sw, x_out, w_out, Cp, y)
    torch.cuda.synchronize()
    check_status(apex)
    rows = np.array([0, 1, 127, 128, g.M // 3, g.M - 1], dtype=np.int64)
    x_in, x_out_ref = oracle.split_outlier_channels(a[rows], ch)
    ap, sa = oracle.quantize_pack(x_in, 128)
    wp, swr = oracle.quantize_pack(w, 128)
    ref = oracle.gemm_dual(ap, sa, wp, swr, x_out_ref, np.ascontiguousarray(w[:, ch]),
                           rows.size, g.N, g.K, 128, 128)
    got = host(y)[rows].astype(np.float64)
    assert_close(got, ref)
    exact = a[rows].astype(np.float64) @ w.astype(np.float64).T
    ap1, sa1 = oracle.quantize_pack(a[rows], 128)
    single = oracle.gemm(ap1, sa1, wp, swr, rows.size, g.N, g.K, 128, 128)
    assert np.abs(got - exact).mean() < 0.5 * np.abs(single - exact).mean()


# ------------------------------------------------------------------ quantized output


def codes_to_q(codes):
    """E4M3 codes of integers -> int64 values (torch's float8_e4m3fn decoding)."""
    t = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy().astype(np.int64)


@pytest.mark.parametrize("M,N,K,gw", [(16, 256, 512, 128), (1, 128, 128, 128),
                                      (129, 384, 1024, 128), (300, 1024, 1152, 384),
                                      (200, 640, 2048, 2048), (1100, 2048, 1024, 128)])
def test_gemm_fp8_quantized_output_is_the_quantizer_of_y(apex, M, N, K, gw):
    """The fused output equals the oracle's activation quantizer applied to the fp16 Y the
    same call wrote, as E4M3 codes and fp16 scales, bit for bit; Y meets the GEMM bar; and
    without Y the quantized output is the same."""
    x = synth.activations(M, K, "outlier", 60 + M)
    w = synth.weights(N, K, 60 + N)
    ac, sa = apex.quantize_act_fp8(dev(x), 128)
    wc, sw = apex.pack_weights_fp8(dev(w), gw)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    yq = torch.empty((M, N), dtype=torch.uint8, device="cuda")
    ys = torch.empty((M, N // 128), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8_quant(M, N, K, 128, gw, ac, sa, wc, sw, y, yq, ys)
    torch.cuda.synchronize()
    check_status(apex)
    ap, sar = oracle.quantize_pack(x, 128)
    wp, swr = oracle.quantize_pack(w, gw)
    y_h = host(y)
    assert_close(y_h.astype(np.float64), oracle.gemm(ap, sar, wp, swr, M, N, K, 128, gw))
    q_ref, s_ref = oracle.quantize_pack(y_h, 128)
    assert np.array_equal(host(yq), e4m3_codes(oracle.unpack(q_ref, N)))
    assert np.array_equal(host(ys).view(np.uint16), s_ref.view(np.uint16))
    yq2, ys2 = torch.zeros_like(yq), torch.zeros_like(ys)
    apex.apex_w4a4_gemm_fp8_quant(M, N, K, 128, gw, ac, sa, wc, sw, None, yq2, ys2)
    torch.cuda.synchronize()
    check_status(apex)
    assert torch.equal(yq2, yq) and torch.equal(ys2, ys)


def test_fp8_chained_layers_through_the_quantized_output(apex):
    """Two W4A4 layers on the E4M3 path, the first one's quantized output fed straight to the
    second: the second's result equals the oracle GEMM on the operands the first produced."""
    M, K, H, N = 256, 1024, 2048, 512
    x = synth.activations(M, K, "student_t", 223)
    w1, w2 = synth.weights(H, K, 224), synth.weights(N, H, 225)
    ac, sa = apex.quantize_act_fp8(dev(x), 128)
    w1c, w1s = apex.pack_weights_fp8(dev(w1), 128)
    w2c, w2s = apex.pack_weights_fp8(dev(w2), 128)
    hq = torch.empty((M, H), dtype=torch.uint8, device="cuda")
    hs = torch.empty((M, H // 128), dtype=torch.float16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    apex.apex_w4a4_gemm_fp8_quant(M, H, K, 128, 128, ac, sa, w1c, w1s, None, hq, hs)
    apex.apex_w4a4_gemm_fp8(M, N, H, 128, 128, hq, hs, w2c, w2s, y)
    torch.cuda.synchronize()
    check_status(apex)
    w2p, w2sr = oracle.quantize_pack(w2, 128)
    ref = oracle.gemm(pack(codes_to_q(host(hq))), host(hs), w2p, w2sr, M, N, H, 128, 128)
    assert_close(host(y).astype(np.float64), ref)


def test_gemm_fp8_quant_argument_rules(apex):
    t = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    h = torch.zeros(1 << 10, dtype=torch.float16, device="cuda")
    with pytest.raises(apex.ApexError) as e:      # N not a multiple of 128
        apex.apex_w4a4_gemm_fp8_quant(16, 200, 256, 128, 128, t, h, t, h, None, t, h)
    assert e.value.code == apex.APEX_ERR_UNSUPPORTED
    with pytest.raises(apex.ApexError) as e:      # no quantized output buffer
        apex.apex_w4a4_gemm_fp8_quant(16, 256, 256, 128, 128, t, h, t, h, None, None, h)
    assert e.value.code == apex.APEX_ERR_INVALID_ARG
