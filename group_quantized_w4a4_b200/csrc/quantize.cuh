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

// One value (an fp16 value widened to fp32) against scale sf (fp32 copy of the stored fp16
// scale): clamp(round_half_even(f / sf), -8, 7), 0 when sf == 0.
__device__ __forceinline__ int quant1(float f, float sf) {
  if (sf == 0.0f) return 0;
  const int q = __float2int_rn(__fdiv_rn(f, sf));
  return min(max(q, -8), 7);
}

// Quantize 8 fp16 values against scale sf and pack them into 4 bytes (little-endian:
// element 0 in the low nibble of byte 0).
__device__ __forceinline__ uint32_t quant_pack8(const uint4& v, float sf) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    const int q0 = quant1(f.x, sf), q1 = quant1(f.y, sf);
    out |= ((uint32_t)(q0 & 0xF) | ((uint32_t)(q1 & 0xF) << 4)) << (8 * i);
  }
  return out;
}

// The same 8 values as 16*q in signed bytes, in the GEMM's operand order: bytes 0..3 hold
// elements 0,2,4,6 and bytes 4..7 elements 1,3,5,7 (what the GEMM makes of a packed word).
__device__ __forceinline__ uint2 quant_expand8(const uint4& v, float sf) {
  const uint32_t w = quant_pack8(v, sf);
  return make_uint2((w << 4) & 0xF0F0F0F0u, w & 0xF0F0F0F0u);
}

// CH > 0: the group is exactly CH 128-wide chunks, kept in registers (one pass over HBM).
// CH == 0: any group width; absmax pass then quantize pass (the second pass hits L2).
// EXP: write the expanded operand form ([rows][K] bytes of 16*q, see quant_expand8)
// instead of packed nibbles ([rows][K/2] bytes).
template <int CH, bool EXP = false>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const __half* __restrict__ x,
                                                            int64_t rows, int64_t K, int group,
                                                            uint8_t* __restrict__ packed,
                                                            __half* __restrict__ scales) {
  // launched as a programmatic dependent: nothing is read or written before the previous
  // grid in the stream has completed
  grid_dep_wait();
  grid_dep_launch();
  const int64_t G = K / group;
  const int64_t units = rows * G;
  const int chunks = group / 128;
  const int lane16 = threadIdx.x & 15;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int half = (threadIdx.x >> 4) & 1;

  // Warp-uniform loop: both half-warps iterate together so the shuffles stay converged.
  for (int64_t base = warp_global * 2; base < units; base += warps_total * 2) {
    const int64_t unit = base + half;
    const bool live = unit < units;
    const int64_t row = live ? unit / G : 0;
    const int64_t g = live ? unit % G : 0;
    const uint4* src = reinterpret_cast<const uint4*>(x + row * K + g * group) + lane16;
    uint32_t* dst =
        reinterpret_cast<uint32_t*>(packed + row * (K / 2) + g * (group / 2)) + lane16;
    uint2* xdst = reinterpret_cast<uint2*>(packed + row * K + (int64_t)g * group) + lane16;

    float amax = 0.0f;
    if constexpr (CH > 0) {
      uint4 v[CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        v[c] = live ? __ldg(src + c * 16) : make_uint4(0, 0, 0, 0);
        amax = fmaxf(amax, absmax8(v[c]));
      }
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s = group_scale(amax);
      const float sf = __half2float(s);
      if (live) {
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          if constexpr (EXP)
            xdst[c * 16] = quant_expand8(v[c], sf);
          else
            dst[c * 16] = quant_pack8(v[c], sf);
        }
        if (lane16 == 0) scales[row * G + g] = s;
      }
    } else {
      for (int c = 0; c < chunks; ++c) {
        uint4 v = live ? __ldg(src + c * 16) : make_uint4(0, 0, 0, 0);
        amax = fmaxf(amax, absmax8(v));
      }
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const __half s = group_scale(amax);
      const float sf = __half2float(s);
      if (live) {
        for (int c = 0; c < chunks; ++c) {
          if constexpr (EXP)
            xdst[c * 16] = quant_expand8(__ldg(src + c * 16), sf);
          else
            dst[c * 16] = quant_pack8(__ldg(src + c * 16), sf);
        }
        if (lane16 == 0) scales[row * G + g] = s;
      }
    }
  }
}

}  // namespace apex
