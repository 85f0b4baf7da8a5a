// dual.cuh -- the inputs of the outlier dual path: a fixed set of input channels (the same for
// every token) bypasses 4-bit quantization and is multiplied in 16 bits.
//
// Method: "OSC: Hardware Efficient W4A4 Quantization via Outlier Separation in Channel
// Dimension" (abstract): outliers sit in fixed channels across tokens; those channels are
// identified offline, gathered online into a compact dense tensor and multiplied in 16 bits,
// beside the 4-bit GEMM of the rest.  Here:
//   * quantize_dual_kernel: the activation quantizer with the outlier channels copied out to
//     x_out [rows][Cp] fp16 (channel order of the list, zero padding up to Cp) and set to zero
//     before the group absmax, so they do not set the 4-bit scales;
//   * gather_columns_kernel: the weights' outlier columns, w_out [N][Cp] fp16 (offline).
// The 16-bit product x_out . w_out^T runs inside the E4M3-carrier GEMM as extra K-steps of
// each tile (gemm_f8.cuh), added to the fp32 accumulators before the single fp16 rounding.
// The channel list is sorted ascending, distinct, each in [0, K) (the caller's contract;
// entries outside a lane's range are skipped, so a bad list gives wrong values, never an
// out-of-bounds access).
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "quantize.cuh"

namespace apex {

// First index i in [0, C) with ch[i] >= k (C when there is none).
__device__ __forceinline__ int lower_bound_ch(const int32_t* __restrict__ ch, int C, int k) {
  int lo = 0, hi = C;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(ch + mid) < k) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// The fp16 bit pattern of element j (0..7) of 8 packed halves.
__device__ __forceinline__ uint16_t half_bits_of(const uint4& v, int j) {
  const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
  return (uint16_t)((j & 1) ? (w >> 16) : (w & 0xFFFFu));
}

// Clear the halves of v whose bit is set in m8.
__device__ __forceinline__ void clear_halves(uint4& v, uint32_t m8) {
  auto keep = [&](int i) {
    return ((m8 >> (2 * i)) & 1u ? 0u : 0x0000FFFFu) |
           ((m8 >> (2 * i + 1)) & 1u ? 0u : 0xFFFF0000u);
  };
  v.x &= keep(0);
  v.y &= keep(1);
  v.z &= keep(2);
  v.w &= keep(3);
}

// One half-warp per (row, 128-wide group), as quantize_pack_kernel<1, FORM>; each lane owns 8
// consecutive channels.  Outlier channels of the lane are found in the sorted list (binary
// search for the lane's first channel, then a short scan).
template <int FORM>
__global__ void __launch_bounds__(128) quantize_dual_kernel(
    const __half* __restrict__ x, int64_t rows, int64_t K, const int32_t* __restrict__ ch,
    int C, uint8_t* __restrict__ out, __half* __restrict__ scales,
    __half* __restrict__ x_out, int Cp) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t G = K / 128;
  const int64_t units = rows * G;
  const int lane16 = threadIdx.x & 15;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int half = (threadIdx.x >> 4) & 1;
  uint16_t* xo = reinterpret_cast<uint16_t*>(x_out);

  for (int64_t base = warp_global * 2; base < units; base += warps_total * 2) {
    const int64_t unit = base + half;
    const bool live = unit < units;
    const int64_t row = live ? unit / G : 0;
    const int64_t g = live ? unit % G : 0;
    const int k0 = (int)(g * 128) + lane16 * 8;
    uint4 v = live ? __ldg(reinterpret_cast<const uint4*>(x + row * K + k0))
                   : make_uint4(0, 0, 0, 0);
    if (live) {
      uint32_t m8 = 0;
      for (int i = lower_bound_ch(ch, C, k0); i < C; ++i) {
        const int k = __ldg(ch + i);
        if (k >= k0 + 8) break;
        if (k < k0) continue;
        xo[row * Cp + i] = half_bits_of(v, k - k0);
        m8 |= 1u << (k - k0);
      }
      clear_halves(v, m8);
      if (g == 0)   // the row's padding columns, once per row
        for (int i = C + lane16; i < Cp; i += 16) xo[row * Cp + i] = 0;
    }
    float amax = absmax8(v);
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const __half s = group_scale(amax);
    const QScale qs = make_qscale(__half2float(s));
    if (live) {
      store_quantized<FORM>(reinterpret_cast<uint32_t*>(out + row * (K / 2) + g * 64) + lane16,
                            reinterpret_cast<uint2*>(out + row * K + g * 128) + lane16, v, qs);
      if (lane16 == 0) scales[row * G + g] = s;
    }
  }
}

// w_out[n][c] = w[n][ch[c]] for c < C, 0 for C <= c < Cp.
__global__ void __launch_bounds__(256) gather_columns_kernel(
    const __half* __restrict__ w, int64_t N, int64_t K, const int32_t* __restrict__ ch, int C,
    __half* __restrict__ w_out, int Cp) {
  grid_dep_wait();
  grid_dep_launch();
  const uint16_t* wb = reinterpret_cast<const uint16_t*>(w);
  uint16_t* ob = reinterpret_cast<uint16_t*>(w_out);
  const int64_t total = N * (int64_t)Cp;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = t / Cp;
    const int c = (int)(t - n * Cp);
    uint16_t v = 0;
    if (c < C) {
      const int k = __ldg(ch + c);
      if (k >= 0 && k < K) v = wb[n * K + k];
    }
    ob[t] = v;
  }
}

}  // namespace apex
