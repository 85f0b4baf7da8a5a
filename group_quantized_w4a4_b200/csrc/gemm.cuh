// gemm.cuh -- W4A4 group-quantized GEMM on sm_100a tensor cores (tcgen05, kind::i8).
//
// Computes Y[m,n] = sum_g P_g[m,n] * sa[m,g] * sw[n, g*128/gw], where
// P_g = sum over the 128-wide K-group g of qa[m,k]*qw[n,k] is an exact integer
// ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing", abstract:
// INT4 tensor-core products with per-group dequantisation on the CUDA cores; the
// mixed-granularity mode keeps 128-wide activation groups and coarser weight groups).
//
// Tile: 128 weight rows (n) x BT tokens (m) per CTA, one K-group (128) per MMA step.
// The MMA runs "weight-stationary": the tensor core's A operand (M = 128) is the weight
// tile held in tensor memory, its B operand (N = BT) the token tile in shared memory, so a
// 16-token decode still uses the full 128-row MMA.  Roles:
//   warp 0      TMA producer: packed W tile [128 x 128 B] and packed A tile [BT x 128 B],
//               two K-groups per stage, into a ring of shared-memory stages (128-byte
//               swizzle).
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma kind::i8 (K = 32 each) per group
//               into a tensor-memory slot; one exact int32 partial per group.
//   warps 2-5   converters: nibbles -> int8 in registers.  The weight row of each thread
//               goes to tensor memory (tcgen05.st); the token rows go to shared memory in
//               the 128-byte-swizzled K-major operand layout.
//   warps 6..   epilogue: tcgen05.ld of a group's partials while the next groups' MMAs
//               run, fp32 scale by sa*sw and accumulate in registers (packed f32x2 math);
//               fp16 output.  Each epilogue thread also fetches the scales it needs, one
//               block of 8 groups ahead (its weight row's sw; one token's sa, shared with
//               the other epilogue threads through a small transposed buffer).
// A warp reaches tensor-memory lanes 32*(warp % 4) .. +31 only, so each group of four
// consecutive warps covers the 128 lanes once (the converter warps 2-5 are lane quarters
// 2,3,0,1; the epilogue warps 6-9 too).
//
// Nibble expansion: for a 32-bit word w of 8 packed nibbles, (w << 4) & 0xF0F0F0F0 holds
// 16*q for the 4 even k and w & 0xF0F0F0F0 16*q for the 4 odd k, as signed bytes.  Both
// operands get the same within-group K order (even k of a word, then odd k), so each
// group's sum is unchanged; the tensor core returns 256*P_g exactly (|256 P_g| <= 2^21),
// and the factor 1/256 is folded into the weight scale.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace apex {

struct GemmArgs {
  int M, N, K;
  int gw;            // weight group (multiple of 128 dividing K)
  int G;             // K / 128
  int Gw;            // K / gw
  int splits;        // K-splits (gridDim.z)
  int gps;           // groups per split
  int sa_vec;        // sa rows readable as 16-byte vectors of 8 groups
  int sw_vec;        // sw rows readable as 16-byte vectors of 8 groups (gw == 128)
  const __half* sa;  // [M][G]
  const __half* sw;  // [N][Gw]
  __half* y;         // [M][N]
  float* ws;         // [splits][M][N] fp32 partial outputs (splits > 1)
  unsigned* counters;  // one arrival counter per output tile (splits > 1)
  int32_t* dump;     // [G][M][N] per-group partials (debug kernel only)
  unsigned long long wait_ns;
  int withhold;      // test hook: the producer never loads this stage (-1: off)
  // Optional timeline trace (null: off), for the first trace_ctas CTAs (linear block id):
  // SM clock stamps (clock64) [cta][role][step] with roles 0 producer issue and 1 converter
  // done (per stage of two K-groups), 2 MMA issued and 3 epilogue done (per K-group);
  // [cta][5][0..1] = %globaltimer at start / end, [cta][5][2] = the SM the CTA ran on,
  // [cta][5][3] = clock64 at start.
  unsigned long long* trace;
  int trace_ctas;
  int trace_steps;
};

__device__ __forceinline__ void trace_stamp(const GemmArgs& a, int role, int step) {
  if (a.trace == nullptr) return;
  const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  if (cta >= a.trace_ctas || step >= a.trace_steps) return;
  a.trace[((size_t)cta * 6 + role) * a.trace_steps + step] =
      role == 5 ? globaltimer_ns() : clock_cycles();
}

template <int BT>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int KPS = 2;                                    // K-groups per packed stage
  static constexpr int NP = BT >= 128 ? 3 : 4;                     // packed stages
  static constexpr int NX = 4;                                     // expanded operand slots
  static constexpr int NSLOT = BT >= 128 ? 3 : (BT >= 64 ? 2 : 4);  // partial (D) slots
  static constexpr int EPI_WARPS = BT >= 128 ? 8 : 4;
  static constexpr int CPT = BT >= 128 ? 64 : BT;  // columns per epilogue thread
  static constexpr int CONV0 = 2;                  // first converter warp
  static constexpr int EPI0 = 6;                   // first epilogue warp
  static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
  static constexpr int MIN_BLOCKS = BT <= 32 ? 2 : 1;  // CTAs per SM the tile is sized for
  static constexpr int W_COL0 = 0;
  static constexpr int D_COL0 = NX * 32;
  static constexpr int TMEM_USED = D_COL0 + NSLOT * BT;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "tensor memory budget");
  static constexpr int PKW = BM * 64 * KPS;   // [BM rows][128 B], 128-byte swizzle
  static constexpr int PKA = BT * 64 * KPS;   // [BT rows][128 B], 128-byte swizzle
  static constexpr int PK_STAGE = PKW + PKA;
  static constexpr int XA = BT * 128;
  static constexpr int SAT = 2 * 8 * BT * 4;  // token scales: 2 blocks x [8 groups][BT] fp32
  static constexpr int OFF_PK = 0;
  static constexpr int OFF_XA = OFF_PK + NP * PK_STAGE;
  static constexpr int OFF_SAT = OFF_XA + NX * XA;
  static constexpr int OFF_BAR = OFF_SAT + SAT;
  static constexpr int NBAR = 2 * NP + 2 * NX + 2 * NSLOT + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(PK_STAGE % 1024 == 0 && XA % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t expand_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t expand_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// The 8 fp16 scales of groups gbeg .. gbeg+7 of one row, as raw bits (zeros from gend on).
// vec: one 16-byte load (row offset + gbeg aligned to 8 elements, weight group == 128).
// Otherwise element loads of base[row_off + g*128/gw].
__device__ __forceinline__ uint4 load_scale_block(const __half* base, size_t row_off, int gbeg,
                                                  int gend, bool vec, int gw) {
  if (vec) return __ldg(reinterpret_cast<const uint4*>(base + row_off + gbeg));
  uint32_t h[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int g = gbeg + j;
    h[j] = g < gend ? __half_as_ushort(base[row_off + (size_t)((g * 128) / gw)]) : 0u;
  }
  return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                    h[6] | (h[7] << 16));
}

__device__ __forceinline__ float half_of(const uint4& v, int j) {
  const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
  return __half2float(__ushort_as_half((uint16_t)((j & 1) ? (w >> 16) : (w & 0xFFFFu))));
}

template <int BT, bool DUMP>
__global__ void __launch_bounds__(GemmCfg<BT>::THREADS, GemmCfg<BT>::MIN_BLOCKS)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmA, const GemmArgs args) {
  using C = GemmCfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pk = smem + C::OFF_PK;
  uint8_t* xa = smem + C::OFF_XA;
  float* s_sat = reinterpret_cast<float*>(smem + C::OFF_SAT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pk_full = bars;
  uint64_t* pk_empty = pk_full + C::NP;
  uint64_t* x_full = pk_empty + C::NP;
  uint64_t* x_empty = x_full + C::NX;
  uint64_t* d_full = x_empty + C::NX;
  uint64_t* d_empty = d_full + C::NSLOT;
  uint64_t* mma_done = d_empty + C::NSLOT;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* s_abort = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* s_last = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  int* s_never = reinterpret_cast<int*>(smem + C::OFF_MISC + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * C::BM;
  const int m0 = blockIdx.y * BT;
  const int g0 = blockIdx.z * args.gps;
  const int ng = min(args.gps, args.G - g0);
  const int ns = (ng + C::KPS - 1) / C::KPS;   // packed stages of this CTA
  const uint64_t lim = args.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(smem_u32(&pk_full[i]), 1);
      mbar_init(smem_u32(&pk_empty[i]), 4);          // one arrival per converter warp
    }
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(smem_u32(&x_full[i]), 4);
      mbar_init(smem_u32(&x_empty[i]), 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(smem_u32(&d_full[i]), 1);
      mbar_init(smem_u32(&d_empty[i]), C::EPI_WARPS);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(mma_done), 1);
    *s_abort = 0;
    *s_last = 0;
    *s_never = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmA);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(s_tmem);
  volatile int* abort_flag = s_abort;
  volatile int* never = s_never;
  if (threadIdx.x == 0) {
    trace_stamp(args, 5, 0);
    if (args.trace != nullptr && args.trace_steps > 3) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
      if (cta < args.trace_ctas) {
        args.trace[((size_t)cta * 6 + 5) * args.trace_steps + 2] = smid;
        args.trace[((size_t)cta * 6 + 5) * args.trace_steps + 3] = clock_cycles();
      }
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last = -1;
      for (int s = 0; s < ns; ++s) {
        const int st = s % C::NP;
        if (!mbar_wait(smem_u32(&pk_empty[st]), ((uint32_t)(s / C::NP) & 1u) ^ 1u, lim,
                       abort_flag))
          break;
        if (s == args.withhold) continue;
        const uint32_t fb = smem_u32(&pk_full[st]);
        const int x = (g0 + s * C::KPS) * 64;   // byte column of the stage's first group
        mbar_arrive_expect_tx(fb, C::PK_STAGE);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE), &tmW, fb, x, n0);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE + C::PKW), &tmA, fb, x, m0);
        trace_stamp(args, 0, s);
        last = s;
      }
      // Never leave the CTA with bulk copies in flight: wait for the last stages issued.
      for (int s = (last - C::NP + 1 > 0 ? last - C::NP + 1 : 0); s <= last; ++s) {
        if (s == args.withhold) continue;
        mbar_wait(smem_u32(&pk_full[s % C::NP]), (uint32_t)(s / C::NP) & 1u, lim, never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, BT);
      for (int i = 0; i < ng; ++i) {
        const int xs = i % C::NX;
        const int sl = i % C::NSLOT;
        if (!mbar_wait(smem_u32(&x_full[xs]), (uint32_t)(i / C::NX) & 1u, lim, abort_flag)) break;
        if (!mbar_wait(smem_u32(&d_empty[sl]), ((uint32_t)(i / C::NSLOT) & 1u) ^ 1u, lim,
                       abort_flag))
          break;
        tc_fence_after();
        const uint32_t a0 = tbase + C::W_COL0 + xs * 32;
        const uint32_t d = tbase + C::D_COL0 + sl * BT;
        const uint64_t b0 = smem_desc_k_sw128(smem_u32(xa + xs * C::XA));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          umma_i8_ts(d, a0 + j * 8, b0 + (uint64_t)(j * 2), idesc, j > 0 ? 1u : 0u);
        umma_commit(smem_u32(&x_empty[xs]));
        umma_commit(smem_u32(&d_full[sl]));
        trace_stamp(args, 2, i);
      }
      umma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0u, lim, never);
    }
  } else if (warp >= C::CONV0 && warp < C::CONV0 + 4) {
    // ------------------------------------------------------------ converters
    const int row = 32 * (warp & 3) + lane;            // this thread's TMEM lane = W row
    const int ct = threadIdx.x - 32 * C::CONV0;        // 0..127, for the token rows
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    constexpr int NIT = C::KPS * BT * 8 / 128;         // token 8-byte units per thread
    for (int s = 0; s < ns; ++s) {
      const int st = s % C::NP;
      const int i0 = s * C::KPS;
      const int nk = min(C::KPS, ng - i0);   // groups of this stage inside the split
      bool ok = mbar_wait(smem_u32(&pk_full[st]), (uint32_t)(s / C::NP) & 1u, lim, abort_flag);
      for (int j = 0; j < nk; ++j)
        ok = ok && mbar_wait(smem_u32(&x_empty[(i0 + j) % C::NX]),
                             ((uint32_t)((i0 + j) / C::NX) & 1u) ^ 1u, lim, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* pw = pk + st * C::PK_STAGE;
      const uint8_t* pa = pw + C::PKW;
      // All shared-memory reads of the stage first, so their latencies overlap.
      uint4 wraw[8];   // this thread's weight row: 16-byte chunk c sits at c ^ (row & 7)
#pragma unroll
      for (int c = 0; c < 8; ++c)
        wraw[c] = *reinterpret_cast<const uint4*>(pw + row * 128 + ((c ^ (row & 7)) << 4));
      uint2 araw[NIT];
#pragma unroll
      for (int q = 0; q < NIT; ++q) {
        const int it = ct + 128 * q;
        const int j = it / (BT * 8), rem = it % (BT * 8);
        const int r = rem >> 3, u = rem & 7;
        araw[q] = *reinterpret_cast<const uint2*>(
            pa + r * 128 + (((4 * j + (u >> 1)) ^ (r & 7)) << 4) + ((u & 1) << 3));
      }
#pragma unroll
      for (int j = 0; j < C::KPS; ++j) {
        if (j < nk) {
          const int xs = (i0 + j) % C::NX;
          uint32_t e0[16], e1[16];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 a = wraw[4 * j + c], b = wraw[4 * j + 2 + c];
            e0[8 * c + 0] = expand_lo(a.x); e0[8 * c + 1] = expand_hi(a.x);
            e0[8 * c + 2] = expand_lo(a.y); e0[8 * c + 3] = expand_hi(a.y);
            e0[8 * c + 4] = expand_lo(a.z); e0[8 * c + 5] = expand_hi(a.z);
            e0[8 * c + 6] = expand_lo(a.w); e0[8 * c + 7] = expand_hi(a.w);
            e1[8 * c + 0] = expand_lo(b.x); e1[8 * c + 1] = expand_hi(b.x);
            e1[8 * c + 2] = expand_lo(b.y); e1[8 * c + 3] = expand_hi(b.y);
            e1[8 * c + 4] = expand_lo(b.z); e1[8 * c + 5] = expand_hi(b.z);
            e1[8 * c + 6] = expand_lo(b.w); e1[8 * c + 7] = expand_hi(b.w);
          }
          const uint32_t tw = tbase + t_lane + C::W_COL0 + xs * 32;
          tmem_st16(tw, e0);
          tmem_st16(tw + 16, e1);
        }
      }
#pragma unroll
      for (int q = 0; q < NIT; ++q) {
        const int it = ct + 128 * q;
        const int j = it / (BT * 8), rem = it % (BT * 8);
        const int r = rem >> 3, u = rem & 7;
        if (j < nk) {
          uint4 o;
          o.x = expand_lo(araw[q].x);
          o.y = expand_hi(araw[q].x);
          o.z = expand_lo(araw[q].y);
          o.w = expand_hi(araw[q].y);
          *reinterpret_cast<uint4*>(xa + ((i0 + j) % C::NX) * C::XA + r * 128 +
                                    ((u ^ (r & 7)) << 4)) = o;
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&pk_empty[st]));
        for (int j = 0; j < nk; ++j) mbar_arrive(smem_u32(&x_full[(i0 + j) % C::NX]));
      }
      if (threadIdx.x == 32 * C::CONV0) trace_stamp(args, 1, s);
    }
  } else if (warp >= C::EPI0) {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 32 * C::EPI0;
    const int h = (warp - C::EPI0) >> 2;           // column block (64 columns) of this warp
    const int row = 32 * (warp & 3) + lane;        // TMEM lane = weight row in the tile
    const int n = n0 + row;
    const bool nvalid = n < args.N;
    const int mt = m0 + et;                        // token whose scales this thread fetches
    const bool tvalid = et < BT && mt < args.M;
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    constexpr int NE = C::EPI_WARPS * 32;
    const int M = args.M, N = args.N;
    // One weight group spans this CTA's whole K-range: sw factors out of the sum.
    const bool hoist = (g0 * 128) / args.gw == ((g0 + ng - 1) * 128) / args.gw;
    const int nblk = (ng + 7) / 8;
    const bool sa_vec = args.sa_vec != 0, sw_vec = args.sw_vec != 0;

    auto sa_block = [&](int b) -> uint4 {
      if (DUMP || !tvalid) return make_uint4(0, 0, 0, 0);
      return load_scale_block(args.sa, (size_t)mt * args.G, g0 + 8 * b, g0 + ng, sa_vec, 128);
    };
    auto sw_block = [&](int b) -> uint4 {
      if (DUMP || !nvalid) return make_uint4(0, 0, 0, 0);
      return load_scale_block(args.sw, (size_t)n * args.Gw, g0 + 8 * b, g0 + ng, sw_vec,
                              args.gw);
    };

    float2 acc[C::CPT / 2];
#pragma unroll
    for (int e = 0; e < C::CPT / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
    float sw_hoisted = 0.0f;

    uint4 sa_c = sa_block(0), sw_c = sw_block(0);
    bool ok = true, aborted = false;
    for (int b = 0; b < nblk; ++b) {
      uint4 sa_n = make_uint4(0, 0, 0, 0), sw_n = make_uint4(0, 0, 0, 0);
      if (b + 1 < nblk) {   // the next block's scales are in flight during this block
        sa_n = sa_block(b + 1);
        sw_n = sw_block(b + 1);
      }
      float* sat = s_sat + (b & 1) * 8 * BT;
      if (et < BT) {
#pragma unroll
        for (int j = 0; j < 8; ++j) sat[j * BT + et] = half_of(sa_c, j);
      }
      aborted = bar_red_or(1, NE, !ok);   // token scales visible; one abort decision for all
      if (aborted) break;
      if (b == 0) sw_hoisted = half_of(sw_c, 0) * (1.0f / 256.0f);
#pragma unroll 1
      for (int j = 0; j < 8; ++j) {
        const int i = 8 * b + j;
        if (i >= ng || !ok) break;
        const int sl = i % C::NSLOT;
        ok = mbar_wait(smem_u32(&d_full[sl]), (uint32_t)(i / C::NSLOT) & 1u, lim, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float4* sab = reinterpret_cast<const float4*>(sat + j * BT + h * 64);
        const float swj = half_of(sw_c, j) * (1.0f / 256.0f);
        const float2 sw2 = make_float2(swj, swj);
        const uint32_t td = tbase + t_lane + C::D_COL0 + sl * BT + h * 64;
#pragma unroll
        for (int cc = 0; cc < C::CPT / 16; ++cc) {
          uint32_t p[16];
          tmem_ld16(td + cc * 16, p);
          if constexpr (DUMP) {
            const int g = g0 + i;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int m = m0 + h * 64 + cc * 16 + e;
              if (m < M && nvalid)
                args.dump[((size_t)g * M + m) * N + n] = static_cast<int32_t>(p[e]) >> 8;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 s4 = sab[cc * 4 + q];
              const float2 pa = make_float2((float)(int32_t)p[4 * q + 0], (float)(int32_t)p[4 * q + 1]);
              const float2 pb = make_float2((float)(int32_t)p[4 * q + 2], (float)(int32_t)p[4 * q + 3]);
              float2 sa_a = make_float2(s4.x, s4.y), sa_b = make_float2(s4.z, s4.w);
              if (!hoist) {
                sa_a = __fmul2_rn(sa_a, sw2);
                sa_b = __fmul2_rn(sa_b, sw2);
              }
              acc[cc * 8 + 2 * q] = __ffma2_rn(pa, sa_a, acc[cc * 8 + 2 * q]);
              acc[cc * 8 + 2 * q + 1] = __ffma2_rn(pb, sa_b, acc[cc * 8 + 2 * q + 1]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&d_empty[sl]));
          if (et == 0) trace_stamp(args, 3, i);
        }
      }
      sa_c = sa_n;
      sw_c = sw_n;
    }
    if (!aborted) aborted = bar_red_or(1, NE, !ok);

    if constexpr (!DUMP) {
      if (!aborted) {
        if (hoist) {
          const float2 sh = make_float2(sw_hoisted, sw_hoisted);
#pragma unroll
          for (int e = 0; e < C::CPT / 2; ++e) acc[e] = __fmul2_rn(acc[e], sh);
        }
        if (args.splits == 1) {
#pragma unroll
          for (int e = 0; e < C::CPT; ++e) {
            const int m = m0 + h * 64 + e;
            const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
            if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(v);
          }
        } else {
          float* wsp = args.ws + (size_t)blockIdx.z * M * N;
#pragma unroll
          for (int e = 0; e < C::CPT; ++e) {
            const int m = m0 + h * 64 + e;
            const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
            if (m < M && nvalid) wsp[(size_t)m * N + n] = v;
          }
          __threadfence();
          bar_red_or(1, NE, false);
          const int tile = blockIdx.y * gridDim.x + blockIdx.x;
          if (et == 0) {
            const unsigned old = atomicAdd(&args.counters[tile], 1u);
            *reinterpret_cast<volatile int*>(s_last) = (old == (unsigned)args.splits - 1u);
          }
          bar_red_or(1, NE, false);
          if (*reinterpret_cast<volatile int*>(s_last)) {
            __threadfence();
            // Sum the splits in split order (deterministic), 16 columns at a time with all
            // of a split's loads issued before they are added.
#pragma unroll
            for (int e0 = 0; e0 < C::CPT; e0 += 16) {
              float sum[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) sum[e] = 0.0f;
              for (int z = 0; z < args.splits; ++z) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const int m = m0 + h * 64 + e0 + e;
                  v[e] = (m < M && nvalid) ? __ldcg(args.ws + ((size_t)z * M + m) * N + n) : 0.0f;
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) sum[e] += v[e];
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int m = m0 + h * 64 + e0 + e;
                if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(sum[e]);
              }
            }
            if (et == 0) atomicExch(&args.counters[tile], 0u);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_stamp(args, 5, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace apex
