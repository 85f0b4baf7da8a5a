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
// entries outside [0, K) are skipped and indices past the list are never written, so a bad
// list gives wrong values, never an out-of-bounds access).
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "quantize.cuh"

namespace apex {

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

// Shared-memory bytes of quantize_dual_kernel's outlier table for K channels.
__host__ __device__ constexpr size_t dual_table_bytes(int64_t K) { return (size_t)(K / 8) * 3; }

// One half-warp per (row, 128-wide group), as quantize_pack_kernel<1, FORM>; each lane owns 8
// consecutive channels (a chunk).  Each block first turns the sorted channel list into a
// table in shared memory: per chunk, a byte with the chunk's outlier channels set, and the
// list index of its first outlier; a lane then finds its outliers with one lookup.  Units
// are indexed in 32 bits (the host launches this kernel only when rows * K / 128 < 2^31),
// split into (row, group) by a shift when K / 128 is a power of two (g_shift >= 0).
template <int FORM>
__global__ void __launch_bounds__(128) quantize_dual_kernel(
    const __half* __restrict__ x, int64_t rows, int64_t K, const int32_t* __restrict__ ch,
    int C, uint8_t* __restrict__ out, __half* __restrict__ scales,
    __half* __restrict__ x_out, int Cp, int g_shift) {
  extern __shared__ uint32_t s_tab[];
  const uint32_t nchunk = (uint32_t)(K / 8);
  uint32_t* s_mask = s_tab;                                           // [nchunk / 4]
  uint16_t* s_first = reinterpret_cast<uint16_t*>(s_tab + nchunk / 4);  // [nchunk]
  grid_dep_wait();
  grid_dep_launch();
  for (uint32_t w = threadIdx.x; w < nchunk / 4; w += blockDim.x) s_mask[w] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < C; i += blockDim.x) {
    const int k = __ldg(ch + i);
    if (k < 0 || k >= K) continue;
    const uint32_t c = (uint32_t)k >> 3;
    atomicOr(&s_mask[c >> 2], 1u << (8 * (c & 3) + (k & 7)));
    if (i == 0 || (uint32_t)(__ldg(ch + i - 1) >> 3) != c) s_first[c] = (uint16_t)i;
  }
  __syncthreads();

  const uint32_t G = (uint32_t)(K / 128);
  const uint32_t units = (uint32_t)(rows * G);
  const int lane16 = threadIdx.x & 15;
  const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t warps_total = (gridDim.x * blockDim.x) >> 5;
  const int half = (threadIdx.x >> 4) & 1;
  uint16_t* xo = reinterpret_cast<uint16_t*>(x_out);

  for (uint32_t base = warp_global * 2; base < units; base += warps_total * 2) {
    const uint32_t unit = base + half;
    const bool live = unit < units;
    const uint32_t u = live ? unit : 0u;
    const uint32_t row = g_shift >= 0 ? u >> g_shift : u / G;
    const uint32_t g = g_shift >= 0 ? u & (G - 1) : u - row * G;
    const uint32_t c = g * 16 + lane16;                      // this lane's chunk
    uint4 v = live ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)row * K) + c)
                   : make_uint4(0, 0, 0, 0);
    if (live) {
      const uint32_t m8 = (s_mask[c >> 2] >> (8 * (c & 3))) & 0xFFu;
      if (m8) {
        uint32_t i = s_first[c];
        for (uint32_t b = m8; b; b &= b - 1, ++i)
          if (i < (uint32_t)C) xo[(size_t)row * Cp + i] = half_bits_of(v, __ffs(b) - 1);
        clear_halves(v, m8);
      }
      if (g == 0)   // the row's padding columns, once per row
        for (int i = C + lane16; i < Cp; i += 16) xo[(size_t)row * Cp + i] = 0;
    }
    float amax = absmax8(v);
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const __half s = group_scale(amax);
    const QScale qs = make_qscale(__half2float(s));
    if (live) {
      store_quantized<FORM>(
          reinterpret_cast<uint32_t*>(out + (size_t)row * (K / 2) + (size_t)g * 64) + lane16,
          reinterpret_cast<uint2*>(out + (size_t)row * K + (size_t)g * 128) + lane16, v, qs);
      if (lane16 == 0) scales[(size_t)row * G + g] = s;
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
