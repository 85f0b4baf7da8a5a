"""GPU parity of the activation quantizer's fast per-value path (batches of 32,768 or more
(row, group) units), on inputs built to land on and next to rounding boundaries, so that the
exact-rule fallback near half-integers runs for many values.

Bar ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing", abstract:
per-token, per-128-group int4 activations): packed bytes, expanded bytes, E4M3 codes and
fp16 scales bit-exact against the oracle's quantizer.
"""
import numpy as np
import pytest

import oracle
from group_quantized_w4a4_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROWS, K = 512, 8192          # 512 x 64 = 32,768 units: the fast path's threshold


@pytest.fixture(scope="module")
def apex():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import group_quantized_w4a4_b200 as m
    m.load_library()
    return m


def boundary_rows(seed):
    """fp16 [ROWS, K]: each 128-wide group has its absmax at 7*s for a power-of-two scale s
    (so s is stored exactly), and its other values at exact ties (k + 1/2)*s, one fp16 ulp
    either side of them, at integers k*s, or random; a quarter of the groups are random."""
    rng = np.random.default_rng(seed)
    x = synth.activations(ROWS, K, "outlier", seed).astype(np.float32)
    G = K // 128
    for r in range(ROWS):
        for g in range(G):
            kind = (r * G + g) % 4
            if kind == 3:
                continue                                   # random group
            s = np.float32(2.0) ** int(rng.integers(-12, 6))
            k = rng.integers(-8, 7, size=128).astype(np.float32)
            v = (k + np.float32(0.5)) * s                  # exact ties
            if kind == 1:                                  # one ulp either side of a tie
                h = v.astype(np.float16)
                up = rng.random(128) < 0.5
                h = np.where(up, np.nextafter(h, np.float16(np.inf)),
                             np.nextafter(h, np.float16(-np.inf)))
                v = h.astype(np.float32)
            elif kind == 2:                                # integers and ties mixed
                v = np.where(rng.random(128) < 0.5, k * s, v)
            v = np.clip(v, -7 * s, 7 * s)
            v[int(rng.integers(0, 128))] = 7 * s * (1 if rng.random() < 0.5 else -1)
            x[r, g * 128:(g + 1) * 128] = v
    return x.astype(np.float16)


def expected_expanded(q):
    """16*q in the GEMM operand order: per 8 elements, k0,k2,k4,k6 then k1,k3,k5,k7."""
    rows, k = q.shape
    blk = q.reshape(rows, k // 8, 8)
    return (blk[:, :, [0, 2, 4, 6, 1, 3, 5, 7]] * 16).reshape(rows, k).astype(np.int8).view(np.uint8)


def e4m3_codes(q):
    """E4M3 bytes of integer values (torch's float8_e4m3fn conversion)."""
    t = torch.from_numpy(q.astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("seed", [1, 2])
def test_fast_path_matches_the_oracle_on_boundary_values(apex, seed):
    x = boundary_rows(seed)
    ap_ref, sa_ref = oracle.quantize_pack(x, 128)
    q_ref = oracle.unpack(ap_ref, K).astype(np.int64)
    # the inputs sit on the boundaries: about a third of all values are exact ties
    ratio = x.astype(np.float64).reshape(ROWS, -1, 128) / np.maximum(
        sa_ref.astype(np.float64)[:, :, None], 1e-30)
    assert np.mean(np.abs(ratio - np.floor(ratio) - 0.5) == 0) > 0.25
    xd = torch.from_numpy(x).cuda()
    ap, sa = apex.quantize_act(xd, 128)
    q8, sa8 = apex.quantize_act_expanded(xd, 128)
    c8, sac = apex.quantize_act_fp8(xd, 128)
    torch.cuda.synchronize()
    assert apex.apex_get_device_status() == 0
    assert np.array_equal(ap.cpu().numpy(), ap_ref)
    assert np.array_equal(q8.cpu().numpy(), expected_expanded(q_ref))
    assert np.array_equal(c8.cpu().numpy(), e4m3_codes(q_ref))
    for s in (sa, sa8, sac):
        assert np.array_equal(s.cpu().numpy().view(np.uint16), sa_ref.view(np.uint16))
