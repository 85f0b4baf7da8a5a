// gemm.cuh -- W4A4 group-quantized GEMM on sm_100a tensor cores (tcgen05, kind::i8).
//
// Computes Y[m,n] = sum_g P_g[m,n] * sa[m,g] * sw[n, g*128/gw], where
// P_g = sum over the 128-wide K-group g of qa[m,k]*qw[n,k] is an exact integer
// ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing", abstract:
// INT4 tensor-core products with per-group dequantisation on the CUDA cores; the
// mixed-granularity mode keeps 128-wide activation groups and coarser weight groups).
//
// Tile: 128 weight rows (n) x BT tokens (m) per CTA, one K-group (128) per pipeline step.
// The MMA runs "weight-stationary": the tensor core's A operand (M = 128) is the weight
// tile held in tensor memory, its B operand (N = BT) the token tile in shared memory, so a
// 16-token decode still uses the full 128-row MMA.  Roles:
//   warp 0      TMA producer: packed W tile [128 x 64 B] and packed A tile [BT x 64 B] per
//               group into a ring of shared-memory stages (64-byte swizzle).
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma kind::i8 (K = 32 each) per group
//               into a tensor-memory slot; one exact int32 partial per group.
//   warps 2-5   converters: nibbles -> int8 in registers.  The weight row of each thread
//               goes to tensor memory (tcgen05.st); the token rows go to shared memory in
//               the 128-byte-swizzled K-major operand layout.
//   warps 6..   epilogue: tcgen05.ld of a group's partials while the next group's MMAs
//               run, fp32 scale by sa*sw and accumulate in registers; fp16 output.
// A warp reaches tensor-memory lanes 32*(warp % 4) .. +31 only, so each group of four
// consecutive warps covers the 128 lanes once (the converter warps 2-5 and the epilogue
// warps 6-9 are lane quarters 2,3,0,1).
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
  int gw;           // weight group (multiple of 128 dividing K)
  int G;            // K / 128
  int Gw;           // K / gw
  int splits;       // K-splits (gridDim.z)
  int gps;          // groups per split
  const __half* sa;  // [M][G]
  const __half* sw;  // [N][Gw]
  __half* y;         // [M][N]
  float* ws;         // [splits][M][N] fp32 partial outputs (splits > 1)
  unsigned* counters;  // one arrival counter per output tile (splits > 1)
  int32_t* dump;     // [G][M][N] per-group partials (debug kernel only)
  unsigned long long wait_ns;
  int withhold;      // test hook: the producer never loads this step (-1: off)
};

template <int BT>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int NP = BT >= 128 ? 4 : (BT >= 64 ? 6 : 8);  // packed stages
  static constexpr int NX = 4;                                     // expanded stages
  static constexpr int NSLOT = BT >= 128 ? 3 : (BT >= 64 ? 2 : 4);  // partial slots
  static constexpr int EPI_WARPS = BT >= 128 ? 8 : 4;
  static constexpr int CPT = BT >= 128 ? 64 : BT;  // columns per epilogue thread
  static constexpr int CONV0 = 2;  // first converter warp
  static constexpr int EPI0 = 6;   // first epilogue warp
  static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
  static constexpr int MIN_BLOCKS = BT <= 32 ? 2 : 1;  // CTAs per SM the tile is sized for
  static constexpr int W_COL0 = 0;
  static constexpr int D_COL0 = NX * 32;
  static constexpr int TMEM_USED = D_COL0 + NSLOT * BT;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "tensor memory budget");
  static constexpr int PKW = BM * 64;
  static constexpr int PKA = BT * 64;
  static constexpr int PK_STAGE = PKW + PKA;
  static constexpr int XA = BT * 128;
  static constexpr int OFF_PK = 0;
  static constexpr int OFF_XA = OFF_PK + NP * PK_STAGE;
  static constexpr int OFF_SA = OFF_XA + NX * XA;
  static constexpr int OFF_BAR = OFF_SA + 2 * BT * 4;
  static constexpr int NBAR = 2 * NP + 2 * NX + 2 * NSLOT + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(PK_STAGE % 1024 == 0 && XA % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t expand_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t expand_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

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
  float* s_sa = reinterpret_cast<float*>(smem + C::OFF_SA);
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
  const uint64_t lim = args.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(smem_u32(&pk_full[i]), 1);
      mbar_init(smem_u32(&pk_empty[i]), 128);
    }
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(smem_u32(&x_full[i]), 128);
      mbar_init(smem_u32(&x_empty[i]), 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(smem_u32(&d_full[i]), 1);
      mbar_init(smem_u32(&d_empty[i]), C::EPI_WARPS * 32);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last = -1;
      for (int i = 0; i < ng; ++i) {
        const int st = i % C::NP;
        const uint32_t ph = (uint32_t)(i / C::NP) & 1u;
        if (!mbar_wait(smem_u32(&pk_empty[st]), ph ^ 1u, lim, abort_flag)) break;
        if (i == args.withhold) continue;
        const uint32_t fb = smem_u32(&pk_full[st]);
        mbar_arrive_expect_tx(fb, C::PK_STAGE);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE), &tmW, fb, (g0 + i) * 64, n0);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE + C::PKW), &tmA, fb, (g0 + i) * 64, m0);
        last = i;
      }
      // Never leave the CTA with bulk copies in flight: wait for the last stages issued.
      for (int i = (last - C::NP + 1 > 0 ? last - C::NP + 1 : 0); i <= last; ++i) {
        if (i == args.withhold) continue;
        mbar_wait(smem_u32(&pk_full[i % C::NP]), (uint32_t)(i / C::NP) & 1u, lim, never);
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
      }
      umma_commit(smem_u32(mma_done));
      mbar_wait(smem_u32(mma_done), 0u, lim, never);
    }
  } else if (warp >= C::CONV0 && warp < C::CONV0 + 4) {
    // ------------------------------------------------------------ converters
    const int row = 32 * (warp & 3) + lane;            // this thread's TMEM lane = W row
    const int ct = threadIdx.x - 32 * C::CONV0;        // 0..127, for the token rows
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    for (int i = 0; i < ng; ++i) {
      const int st = i % C::NP;
      const int xs = i % C::NX;
      bool ok = mbar_wait(smem_u32(&pk_full[st]), (uint32_t)(i / C::NP) & 1u, lim, abort_flag);
      ok = ok && mbar_wait(smem_u32(&x_empty[xs]), ((uint32_t)(i / C::NX) & 1u) ^ 1u, lim,
                           abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* pw = pk + st * C::PK_STAGE;
      uint32_t wv[16];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 v =
            *reinterpret_cast<const uint4*>(pw + row * 64 + ((c ^ ((row >> 1) & 3)) << 4));
        wv[4 * c + 0] = v.x;
        wv[4 * c + 1] = v.y;
        wv[4 * c + 2] = v.z;
        wv[4 * c + 3] = v.w;
      }
      uint32_t e0[16], e1[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        e0[2 * j] = expand_lo(wv[j]);
        e0[2 * j + 1] = expand_hi(wv[j]);
        e1[2 * j] = expand_lo(wv[8 + j]);
        e1[2 * j + 1] = expand_hi(wv[8 + j]);
      }
      const uint32_t tw = tbase + t_lane + C::W_COL0 + xs * 32;
      tmem_st16(tw, e0);
      tmem_st16(tw + 16, e1);

      const uint8_t* pa = pw + C::PKW;
      uint8_t* xd = xa + xs * C::XA;
#pragma unroll
      for (int it = ct; it < BT * 8; it += 128) {
        const int r = it >> 3, u = it & 7;
        const uint2 v = *reinterpret_cast<const uint2*>(pa + r * 64 +
                                                        (((u >> 1) ^ ((r >> 1) & 3)) << 4) +
                                                        ((u & 1) << 3));
        uint4 o;
        o.x = expand_lo(v.x);
        o.y = expand_hi(v.x);
        o.z = expand_lo(v.y);
        o.w = expand_hi(v.y);
        *reinterpret_cast<uint4*>(xd + r * 128 + ((u ^ (r & 7)) << 4)) = o;
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&pk_empty[st]));
      mbar_arrive(smem_u32(&x_full[xs]));
    }
  } else if (warp >= C::EPI0) {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 32 * C::EPI0;
    const int h = (warp - C::EPI0) >> 2;           // column block (64 columns) of this warp
    const int row = 32 * (warp & 3) + lane;        // TMEM lane = weight row in the tile
    const int n = n0 + row;
    const bool nvalid = n < args.N;
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    constexpr int NE = C::EPI_WARPS * 32;
    const int M = args.M, N = args.N;

    // The partials export has no scales (its launch passes none): never touch them there.
    auto load_sa = [&](int g) -> float {
      if constexpr (DUMP) return 0.0f;
      const int m = m0 + et;
      return (et < BT && m < M) ? __half2float(args.sa[(size_t)m * args.G + g]) : 0.0f;
    };
    auto load_sw = [&](int g) -> float {
      if constexpr (DUMP) return 0.0f;
      return nvalid ? __half2float(args.sw[(size_t)n * args.Gw + (g * 128) / args.gw]) *
                          (1.0f / 256.0f)
                    : 0.0f;
    };

    float acc[C::CPT];
#pragma unroll
    for (int e = 0; e < C::CPT; ++e) acc[e] = 0.0f;

    if (et < BT) s_sa[et] = load_sa(g0);
    float sw_cur = load_sw(g0);
    bool aborted = bar_red_or(1, NE, false);
    for (int i = 0; i < ng && !aborted; ++i) {
      const int g = g0 + i;
      const int sl = i % C::NSLOT;
      const float sa_next = (i + 1 < ng) ? load_sa(g + 1) : 0.0f;
      const float sw_next = (i + 1 < ng) ? load_sw(g + 1) : 0.0f;
      bool ok = mbar_wait(smem_u32(&d_full[sl]), (uint32_t)(i / C::NSLOT) & 1u, lim, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        const float* sab = s_sa + (i & 1) * BT + h * 64;
        const uint32_t td = tbase + t_lane + C::D_COL0 + sl * BT + h * 64;
#pragma unroll
        for (int cc = 0; cc < C::CPT / 16; ++cc) {
          uint32_t p[16];
          tmem_ld16(td + cc * 16, p);
          if constexpr (DUMP) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int m = m0 + h * 64 + cc * 16 + e;
              if (m < M && nvalid)
                args.dump[((size_t)g * M + m) * N + n] = static_cast<int32_t>(p[e]) >> 8;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float s = sab[cc * 16 + e] * sw_cur;
              acc[cc * 16 + e] =
                  fmaf(static_cast<float>(static_cast<int32_t>(p[e])), s, acc[cc * 16 + e]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&d_empty[sl]));
        if (et < BT) s_sa[((i + 1) & 1) * BT + et] = sa_next;
      }
      sw_cur = sw_next;
      aborted = bar_red_or(1, NE, !ok);
    }

    if constexpr (!DUMP) {
      if (!aborted) {
        if (args.splits == 1) {
#pragma unroll
          for (int e = 0; e < C::CPT; ++e) {
            const int m = m0 + h * 64 + e;
            if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(acc[e]);
          }
        } else {
          float* wsp = args.ws + (size_t)blockIdx.z * M * N;
#pragma unroll
          for (int e = 0; e < C::CPT; ++e) {
            const int m = m0 + h * 64 + e;
            if (m < M && nvalid) wsp[(size_t)m * N + n] = acc[e];
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
#pragma unroll 4
            for (int e = 0; e < C::CPT; ++e) {
              const int m = m0 + h * 64 + e;
              if (m < M && nvalid) {
                float s = 0.0f;
                for (int z = 0; z < args.splits; ++z)
                  s += __ldcg(args.ws + ((size_t)z * M + m) * N + n);
                args.y[(size_t)m * N + n] = __float2half_rn(s);
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace apex
