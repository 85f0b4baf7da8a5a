// quantize.cuh -- per-row, per-K-group symmetric int4 quantization and nibble packing.
//
// Method: "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing"
// (abstract): activations and weights are both 4-bit with one scale per 128-wide K-group
// (coarser weight groups in the mixed-granularity mode).  Quantizer rule used here (the
// plainest reading of that statement):
//   s = fp16_rne(fp32(absmax over the group) / 7)            (IEEE fp32 division)
//   q = clamp(round_half_even(fp32(x) / fp32(s)), -8, 7)     (q = 0 when s == 0)
//   byte j of a row = q[2j] in bits 0..3 | q[2j+1] in bits 4..7
//
// Layout of the work: one half-warp (16 threads) owns one (row, group); each thread owns 8
// consecutive K elements of every 128-wide chunk, so the 16 threads read 256 contiguous
// bytes per chunk (one 16-byte load each) and write 64 contiguous packed bytes.  The
// group's absmax is a 4-step xor-shuffle reduction inside the half-warp.  Groups wider
// than 512 are processed in two passes (absmax, then quantize), re-reading the row from
// L2; that only happens for the offline weight packing with coarse groups.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace apex {

__device__ __forceinline__ float absmax8(const uint4& v) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  __half2 m = __hmax2(__habs2(h[0]), __habs2(h[1]));
  m = __hmax2(m, __hmax2(__habs2(h[2]), __habs2(h[3])));
  return fmaxf(__low2float(m), __high2float(m));
}

// The group's stored scale: fp16_rne(fp32(absmax) / 7), IEEE fp32 division.
__device__ __forceinline__ __half group_scale(float absmax) {
  return __float2half_rn(__fdiv_rn(absmax, 7.0f));
}

// A group's stored scale in the form the per-value rule uses: s (fp32 copy of the stored
// fp16 scale), r = 1/s correctly rounded, and s/2 (exact).
struct QScale {
  float s, r, h;
};
__device__ __forceinline__ QScale make_qscale(float sf) {
  QScale q;
  q.s = sf;
  q.r = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
  q.h = 0.5f * sf;
  return q;
}

// One value (an fp16 value widened to fp32): clamp(round_half_even(f / s), -8, 7), 0 when
// s == 0, without a division.  q0 = rne(f * r) is within one of the answer; the residual
// e = f - q0 * s is exact in fp32 for fp16 f and s (one fma), and it decides the last step:
// |e| > s/2 moves q0 one toward e, |e| == s/2 is a tie and moves it only if q0 is odd.
// This equals the correctly rounded quotient's rounding for every (f, s) the quantizer
// meets, which a CPU test checks exhaustively.
__device__ __forceinline__ float quant1f(float f, const QScale& qs) {
  if (qs.s == 0.0f) return 0.0f;
  const float q0 = rintf(__fmul_rn(f, qs.r));
  const float e = __fmaf_rn(-q0, qs.s, f);
  const float ae = fabsf(e);
  const bool odd = (__float2int_rn(q0) & 1) != 0;
  const float q = (ae > qs.h || (ae == qs.h && odd)) ? q0 + copysignf(1.0f, e) : q0;
  return fminf(fmaxf(q, -8.0f), 7.0f);
}

__device__ __forceinline__ int quant1(float f, const QScale& qs) {
  return __float2int_rn(quant1f(f, qs));
}

// Byte permute: byte i of the result is byte sel[4i+3:4i] of the 8 bytes {b, a} (a = 0..3).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// E4M3 codes of the four nibbles (int4 two's complement) in the low 16 bits of w, nibble i
// -> byte i, by two 8-byte table lookups: the codes of q = 0..7 and of q = -8..-1, indexed by
// the nibble's low three bits, the sign bit choosing the table.  E4M3: 1 sign bit, 4
// exponent bits with bias 7, 3 mantissa bits; every q in [-8, 7] is exact and 0 is 0x00.
__device__ __forceinline__ uint32_t e4m3_of_nibbles(uint32_t w) {
  constexpr uint32_t P0 = 0x44403800u, P1 = 0x4E4C4A48u;   // 0, 1, 2, 3 | 4, 5, 6, 7
  constexpr uint32_t N0 = 0xCACCCED0u, N1 = 0xB8C0C4C8u;   // -8,-7,-6,-5 | -4,-3,-2,-1
  const uint32_t idx = w & 0x7777u;
  const uint32_t pos = prmt(P0, P1, idx);
  const uint32_t neg = prmt(N0, N1, idx);
  // 0xFF in byte i where nibble i is negative: selector 0xC (sign of byte 4 = 0x80) or 0x0
  const uint32_t sg = w & 0x8888u;
  const uint32_t mask = prmt(0u, 0x80u, sg | (sg >> 1));
  return (neg & mask) | (pos & ~mask);
}

// The exact rule (quant1) for 8 values, packed as below.
__device__ __forceinline__ uint32_t quant_pack8_exact(const uint4& v, const QScale& qs) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    const int q0 = quant1(f.x, qs), q1 = quant1(f.y, qs);
    out |= ((uint32_t)(q0 & 0xF) | ((uint32_t)(q1 & 0xF) << 4)) << (8 * i);
  }
  return out;
}

// Quantize 8 fp16 values against the group scale qs and pack them into 4 bytes (little-endian:
// element 0 in the low nibble of byte 0).
// Fast path, on the fp32 pipe alone: t = fl(f * r) differs from the exact quotient f / s by
// at most 2^-19 (|f / s| <= 10.5 for every value of a group against its own scale), so
// unless t lies within 2^-18 of a half-integer both round to the same integer.  t, clamped
// to [-8, 7] (clamping and rounding commute), plus 1.5 * 2^23 is that integer rounded to
// nearest even, held in two's complement in the low bits of the sum.  Near a half-integer
// the exact rule decides (under 0.1 % of all reachable (f, s) pairs; a CPU test enumerates
// them all and checks the whole claim).  A zero scale has r = 0, so
// every t is 0; a NaN t clamps to -8, as the exact rule's clamp gives.
// FAST = false: the exact rule alone (a shorter dependency chain, for latency-bound callers).
template <bool FAST = true>
__device__ __forceinline__ uint32_t quant_pack8(const uint4& v, const QScale& qs) {
  if constexpr (!FAST) return quant_pack8_exact(v, qs);
  constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
  constexpr float kNear = 0.5f - 0x1p-18f;
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t y[8];
  bool near = false;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    const float t0 = fminf(fmaxf(__fmul_rn(f.x, qs.r), -8.0f), 7.0f);
    const float t1 = fminf(fmaxf(__fmul_rn(f.y, qs.r), -8.0f), 7.0f);
    const float y0 = __fadd_rn(t0, kMagic), y1 = __fadd_rn(t1, kMagic);
    near |= fabsf(__fsub_rn(t0, __fsub_rn(y0, kMagic))) >= kNear;
    near |= fabsf(__fsub_rn(t1, __fsub_rn(y1, kMagic))) >= kNear;
    y[2 * i] = __float_as_uint(y0);
    y[2 * i + 1] = __float_as_uint(y1);
  }
  if (near) return quant_pack8_exact(v, qs);
  // low bytes: q0 q2 q4 q6 and q1 q3 q5 q7
  const uint32_t ev = prmt(prmt(y[0], y[2], 0x0040u), prmt(y[4], y[6], 0x0040u), 0x5410u);
  const uint32_t od = prmt(prmt(y[1], y[3], 0x0040u), prmt(y[5], y[7], 0x0040u), 0x5410u);
  return (ev & 0x0F0F0F0Fu) | ((od & 0x0F0F0F0Fu) << 4);
}

// The same 8 values as the E4M3 codes of q (one byte per element, in element order): the
// 8-bit float operand form of the tensor cores' kind::f8f6f4, which holds every q in
// [-8, 7] exactly.
template <bool FAST = true>
__device__ __forceinline__ uint2 quant_e4m3_8(const uint4& v, const QScale& qs) {
  const uint32_t w = quant_pack8<FAST>(v, qs);
  return make_uint2(e4m3_of_nibbles(w), e4m3_of_nibbles(w >> 16));
}

// The same 8 values as 16*q in signed bytes, in the GEMM's operand order: bytes 0..3 hold
// elements 0,2,4,6 and bytes 4..7 elements 1,3,5,7 (what the GEMM makes of a packed word).
template <bool FAST = true>
__device__ __forceinline__ uint2 quant_expand8(const uint4& v, const QScale& qs) {
  const uint32_t w = quant_pack8<FAST>(v, qs);
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

// Output forms of the quantizer: packed nibbles ([rows][K/2] bytes), the expanded int8
// operand form ([rows][K] bytes of 16*q, see quant_expand8), or E4M3 codes of q ([rows][K]
// bytes, element order, see quant_e4m3_8).
enum QForm : int { FORM_PACKED = 0, FORM_EXPANDED = 1, FORM_E4M3 = 2 };

template <int FORM, bool FAST = true>
__device__ __forceinline__ void store_quantized(uint32_t* dst, uint2* xdst, const uint4& v,
                                                const QScale& qs) {
  if constexpr (FORM == FORM_EXPANDED)
    *xdst = quant_expand8<FAST>(v, qs);
  else if constexpr (FORM == FORM_E4M3)
    *xdst = quant_e4m3_8<FAST>(v, qs);
  else
    *dst = quant_pack8<FAST>(v, qs);
}

// CH > 0: the group is exactly CH 128-wide chunks, kept in registers (one pass over HBM).
// CH == 0: any group width; absmax pass then quantize pass (the second pass hits L2).
// FORM: the output form (QForm).
// Each half-warp takes UPT (row, group) units per round, all their loads issued before any
// arithmetic, so that several 16-byte loads per thread are in flight (the kernel is bound by
// memory latency, not by its arithmetic).  FAST: the fast per-value path (quant_pack8), for
// throughput; without it the exact rule alone, whose shorter chain suits a batch of a few
// tokens, where each thread quantizes one group and the latency of that chain is the time.
// Units are indexed in 32 bits (the host launches this kernel only when rows * K / group <
// 2^31) and split into (row, group) by a shift when the groups per row are a power of two
// (g_shift >= 0).
template <int CH, int FORM = FORM_PACKED, int UPT = 1, bool FAST = true>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const __half* __restrict__ x,
                                                            int64_t rows, int64_t K, int group,
                                                            uint8_t* __restrict__ packed,
                                                            __half* __restrict__ scales,
                                                            int g_shift) {
  // launched as a programmatic dependent: nothing is read or written before the previous
  // grid in the stream has completed
  grid_dep_wait();
  grid_dep_launch();
  const uint32_t G = (uint32_t)(K / group);
  const uint32_t units = (uint32_t)(rows * G);
  const int chunks = group / 128;
  const int lane16 = threadIdx.x & 15;
  const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t warps_total = (gridDim.x * blockDim.x) >> 5;
  const int half = (threadIdx.x >> 4) & 1;
  auto split = [&](uint32_t unit, uint32_t& row, uint32_t& g) {
    if (g_shift >= 0) {
      row = unit >> g_shift;
      g = unit & (G - 1);
    } else {
      row = unit / G;
      g = unit - row * G;
    }
  };

  // Warp-uniform loop: both half-warps iterate together so the shuffles stay converged.
  for (uint32_t base = warp_global * 2 * UPT; base < units; base += warps_total * 2 * UPT) {
    if constexpr (CH > 0) {
      uint4 v[UPT][CH];
      uint32_t row[UPT], g[UPT];
      bool live[UPT];
#pragma unroll
      for (int u = 0; u < UPT; ++u) {
        const uint32_t unit = base + 2 * u + half;
        live[u] = unit < units;
        split(live[u] ? unit : 0u, row[u], g[u]);
        const uint4* src =
            reinterpret_cast<const uint4*>(x + (int64_t)row[u] * K + (int64_t)g[u] * group) +
            lane16;
#pragma unroll
        for (int c = 0; c < CH; ++c)
          v[u][c] = live[u] ? __ldg(src + c * 16) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < UPT; ++u) {
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < CH; ++c) amax = fmaxf(amax, absmax8(v[u][c]));
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const __half s = group_scale(amax);
        const QScale qs = make_qscale(__half2float(s));
        if (live[u]) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(packed + (int64_t)row[u] * (K / 2) +
                                                      (int64_t)g[u] * (group / 2)) + lane16;
          uint2* xdst = reinterpret_cast<uint2*>(packed + (int64_t)row[u] * K +
                                                 (int64_t)g[u] * group) + lane16;
#pragma unroll
          for (int c = 0; c < CH; ++c)
            store_quantized<FORM, FAST>(dst + c * 16, xdst + c * 16, v[u][c], qs);
          if (lane16 == 0) scales[(int64_t)row[u] * G + g[u]] = s;
        }
      }
    } else {
      const uint32_t unit = base + half;
      const bool live = unit < units;
      uint32_t row, g;
      split(live ? unit : 0u, row, g);
      const uint4* src =
          reinterpret_cast<const uint4*>(x + (int64_t)row * K + (int64_t)g * group) + lane16;
      float amax = 0.0f;
      for (int c = 0; c < chunks; ++c) {
        uint4 v = live ? __ldg(src + c * 16) : make_uint4(0, 0, 0, 0);
        amax = fmaxf(amax, absmax8(v));
      }
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s = group_scale(amax);
      const QScale qs = make_qscale(__half2float(s));
      if (live) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(packed + (int64_t)row * (K / 2) +
                                                    (int64_t)g * (group / 2)) + lane16;
        uint2* xdst =
            reinterpret_cast<uint2*>(packed + (int64_t)row * K + (int64_t)g * group) + lane16;
        for (int c = 0; c < chunks; ++c)
          store_quantized<FORM, FAST>(dst + c * 16, xdst + c * 16, __ldg(src + c * 16), qs);
        if (lane16 == 0) scales[(int64_t)row * G + g] = s;
      }
    }
  }
}

}  // namespace apex
