"""The quantizer's rounding rule, q = clamp(rne(fl32(x / s)), -8, 7), reached without a
division per element: r = fl32(1 / s), q0 = rne(fl32(x * r)), then one exact correction
from the residual e = x - q0 * s (an fma, exact for these operands).  Checked on every
pair the quantizer can meet: every fp16 x with |x| <= absmax and s = fp16(fl32(absmax) / 7)
for every positive finite fp16 absmax.  This is the identity a division-free quantizer
relies on; plain numpy, no GPU.  The same pairs check the quantizer's fast path, which rounds
fl32(x * r) by an fp32 addition and falls back to the exact rule near half-integers."""
import numpy as np


def corrected(x, s):
    r = np.float32(1) / s
    q0 = np.rint(x * r)
    e64 = x.astype(np.float64) - q0.astype(np.float64) * np.float64(s)
    e = e64.astype(np.float32)
    assert np.array_equal(e.astype(np.float64), e64), "the residual is not exact in fp32"
    h = np.float32(0.5) * s
    ae, sg = np.abs(e), np.sign(e)
    q = np.where(ae > h, q0 + sg, q0)
    q = np.where((ae == h) & (np.abs(q0) % 2 == 1), q0 + sg, q)   # a tie goes to even
    return np.clip(q, -8, 7), np.clip(q0, -8, 7)


MAGIC = np.float32(12582912.0)          # 1.5 * 2^23
NEAR = np.float32(0.5 - 2.0 ** -18)


def fast(x, s):
    """The quantizer's fast path: t = fl32(x * r) clamped to [-8, 7], rounded to an integer
    (ties to even) by adding 1.5 * 2^23, whose low bits then hold the integer in two's
    complement.  It is taken unless t lies within 2^-18 of a half-integer ("near"); there the
    exact rule above decides.  Returns (q, its 4-bit code from the sum's bits, near)."""
    r = np.float32(1) / s
    t = np.clip(x * r, np.float32(-8), np.float32(7))
    y = t + MAGIC
    q = y - MAGIC
    near = np.abs(t - q) >= NEAR
    return q, y.view(np.uint32) & np.uint32(0xF), near


def test_division_free_rounding_matches_on_every_reachable_pair():
    nonneg = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    absmax = nonneg[1:]
    scale = (absmax / np.float32(7)).astype(np.float16).astype(np.float32)
    order = np.argsort(scale, kind="stable")
    s_sorted, a_sorted = scale[order], absmax[order]
    uniq, first = np.unique(s_sorted, return_index=True)
    a_max = np.maximum.reduceat(a_sorted, first)   # the widest group each scale serves
    pairs = naive_wrong = near_count = 0
    for s, amx in zip(uniq, a_max):
        s = np.float32(s)
        if s == 0:
            continue        # a zero scale quantizes everything to 0, no division taken
        xp = nonneg[:np.searchsorted(nonneg, amx, side="right")]
        x = np.concatenate([xp, -xp[1:]])
        want = np.clip(np.rint(x / s), -8, 7)
        got, naive = corrected(x, s)
        assert np.array_equal(got, want), f"scale {s}"
        qf, code, near = fast(x, s)
        ok = near | ((qf == want) & (code == (want.astype(np.int32) & 0xF).astype(np.uint32)))
        assert ok.all(), f"fast path, scale {s}"
        pairs += x.size
        naive_wrong += int(np.count_nonzero(naive != want))
        near_count += int(np.count_nonzero(near))
    assert pairs == 888_529_158
    assert naive_wrong > 0     # the correction step is needed, not decoration
    assert near_count < pairs // 1000   # the exact rule is the rare path


def test_correction_handles_ties_to_even():
    s = np.float32(1.0)
    x = np.array([0.5, 1.5, 2.5, -0.5, -1.5, 6.5, 7.0], dtype=np.float32)
    got, _ = corrected(x, s)
    assert got.tolist() == [0.0, 2.0, 2.0, -0.0, -2.0, 6.0, 7.0]
