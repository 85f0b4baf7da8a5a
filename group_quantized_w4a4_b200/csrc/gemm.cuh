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
//   warp 0      TMA producer: packed W tile [128 x 128 B] and packed A tile [BT x 128 B],
//               two K-groups per stage (128-byte rows halve the TMA row requests per
//               byte), into a ring of shared-memory stages (128-byte swizzle).
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma kind::i8 (K = 32 each) per group
//               into a tensor-memory slot; one exact int32 partial per group.
//   warps 2-5   converters: nibbles -> int8 in registers.  The weight row of each thread
//               goes to tensor memory (tcgen05.st); the token rows go to shared memory in
//               the 128-byte-swizzled K-major operand layout.
//   warp 6      scale loader: the fp16 group scales sa (per token) and sw (per weight row)
//               of upcoming groups, converted to fp32 into a shared-memory ring, several
//               groups ahead of their use (their global-load latency is off the critical
//               path).
//   warps 7..   epilogue: tcgen05.ld of a group's partials while the next group's MMAs
//               run, fp32 scale by sa*sw and accumulate in registers (packed f32x2 math);
//               fp16 output.
// A warp reaches tensor-memory lanes 32*(warp % 4) .. +31 only, so each group of four
// consecutive warps covers the 128 lanes once (the converter warps 2-5 are lane quarters
// 2,3,0,1 and the epilogue warps 7-10 quarters 3,0,1,2).
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
  // Optional timeline trace (null: off): for the first trace_ctas CTAs (linear block id),
  // SM clock stamps (clock64) [cta][role][step] with roles 0 producer issue and 1 converter
  // done (per stage of two K-groups), 2 MMA issued, 3 epilogue done and 4 scale loader done
  // (per K-group); [cta][5][0..1] = %globaltimer at start / end, [cta][5][2] = the SM the
  // CTA ran on, [cta][5][3] = clock64 at start.
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
  static constexpr int NX = 4;                                     // expanded stages
  static constexpr int NSLOT = BT >= 128 ? 3 : (BT >= 64 ? 2 : 4);  // partial slots
  static constexpr int SR = 8;                                     // scale ring slots
  static constexpr int SB = 4;                                     // scale loader batch
  static constexpr int EPI_WARPS = BT >= 128 ? 8 : 4;
  static constexpr int CPT = BT >= 128 ? 64 : BT;  // columns per epilogue thread
  static constexpr int CONV0 = 2;  // first converter warp
  static constexpr int LOADER = 6;  // scale loader warp
  static constexpr int EPI0 = 7;   // first epilogue warp
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
  static constexpr int SC_SLOT = (BT + BM) * 4;   // fp32 sa[BT] then sw[BM]
  // Raw scale blocks brought in by TMA: 8 consecutive groups x rows, fp16.
  static constexpr int RS = 3;                     // raw sa blocks in flight
  static constexpr int RW = 2;                     // raw sw blocks in flight
  static constexpr int RSA = BT * 16;
  static constexpr int RSW = BM * 16;
  static constexpr int OFF_PK = 0;
  static constexpr int OFF_XA = OFF_PK + NP * PK_STAGE;
  static constexpr int OFF_SC = OFF_XA + NX * XA;
  static constexpr int OFF_RSA = OFF_SC + SR * SC_SLOT;
  static constexpr int OFF_RSW = OFF_RSA + RS * RSA;
  static constexpr int OFF_BAR = OFF_RSW + RW * RSW;
  static constexpr int NBAR = 2 * NP + 2 * NX + 2 * NSLOT + 2 * SR + 2 * RS + 2 * RW + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(PK_STAGE % 1024 == 0 && XA % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t expand_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t expand_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// SCT: the scales come in by TMA, in blocks of 8 groups ([rows][8] fp16), together with
// the packed data.  That needs row strides that are multiples of 16 bytes: K/128 % 8 == 0
// for sa and K/gw % 8 == 0 for sw (or K/gw == 1: one weight scale per row, read once).
// Otherwise the loader warp reads each group's scales with plain loads.
template <int BT, bool DUMP, bool SCT>
__global__ void __launch_bounds__(GemmCfg<BT>::THREADS, GemmCfg<BT>::MIN_BLOCKS)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmSA,
                     const __grid_constant__ CUtensorMap tmSW, const GemmArgs args) {
  using C = GemmCfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pk = smem + C::OFF_PK;
  uint8_t* xa = smem + C::OFF_XA;
  float* s_sc = reinterpret_cast<float*>(smem + C::OFF_SC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pk_full = bars;
  uint64_t* pk_empty = pk_full + C::NP;
  uint64_t* x_full = pk_empty + C::NP;
  uint64_t* x_empty = x_full + C::NX;
  uint64_t* d_full = x_empty + C::NX;
  uint64_t* d_empty = d_full + C::NSLOT;
  uint64_t* sc_full = d_empty + C::NSLOT;
  uint64_t* sc_empty = sc_full + C::SR;
  uint64_t* rsa_full = sc_empty + C::SR;
  uint64_t* rsa_empty = rsa_full + C::RS;
  uint64_t* rsw_full = rsa_empty + C::RS;
  uint64_t* rsw_empty = rsw_full + C::RW;
  uint64_t* mma_done = rsw_empty + C::RW;
  const uint16_t* rsa = reinterpret_cast<const uint16_t*>(smem + C::OFF_RSA);
  const uint16_t* rsw = reinterpret_cast<const uint16_t*>(smem + C::OFF_RSW);
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
      mbar_init(smem_u32(&pk_empty[i]), 4);             // one arrival per converter warp
    }
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(smem_u32(&x_full[i]), 4);
      mbar_init(smem_u32(&x_empty[i]), 1);
    }
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(smem_u32(&d_full[i]), 1);
      mbar_init(smem_u32(&d_empty[i]), C::EPI_WARPS);   // one arrival per epilogue warp
    }
    for (int i = 0; i < C::SR; ++i) {
      mbar_init(smem_u32(&sc_full[i]), 1);
      mbar_init(smem_u32(&sc_empty[i]), C::EPI_WARPS);
    }
    for (int i = 0; i < C::RS; ++i) {
      mbar_init(smem_u32(&rsa_full[i]), 1);
      mbar_init(smem_u32(&rsa_empty[i]), 1);
    }
    for (int i = 0; i < C::RW; ++i) {
      mbar_init(smem_u32(&rsw_full[i]), 1);
      mbar_init(smem_u32(&rsw_empty[i]), 1);
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
    if constexpr (SCT) {
      tma_prefetch_desc(&tmSA);
      tma_prefetch_desc(&tmSW);
    }
  }
  // weight-scale block (8 weight groups) needed by step i, for the TMA scale path
  auto wblock = [&](int i) { return ((g0 + i) * 128 / args.gw) >> 3; };
  const bool sw_tma = SCT && args.Gw % 8 == 0;
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(s_tmem);
  if (threadIdx.x == 0) {
    trace_stamp(args, 5, 0);
    if (args.trace != nullptr && args.trace_steps > 2) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      const int cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
      if (cta < args.trace_ctas) {
        args.trace[((size_t)cta * 6 + 5) * args.trace_steps + 2] = smid;
        if (args.trace_steps > 3)
          args.trace[((size_t)cta * 6 + 5) * args.trace_steps + 3] = clock_cycles();
      }
    }
  }
  volatile int* abort_flag = s_abort;
  volatile int* never = s_never;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int last = -1, last_sa = -1, last_sw = -1;   // last issued blocks (for the drain)
      const int ns = (ng + C::KPS - 1) / C::KPS;
      for (int sidx = 0; sidx < ns; ++sidx) {
        const int i = sidx * C::KPS;      // first K-group of the stage
        const int st = sidx % C::NP;
        const uint32_t ph = (uint32_t)(sidx / C::NP) & 1u;
        if (!mbar_wait(smem_u32(&pk_empty[st]), ph ^ 1u, lim, abort_flag)) break;
        if (sidx == args.withhold) continue;
        if constexpr (SCT && !DUMP) {
          if ((i & 7) == 0) {   // the split starts on a multiple of 8 groups
            const int b = i >> 3, rs = b % C::RS;
            if (!mbar_wait(smem_u32(&rsa_empty[rs]), ((uint32_t)(b / C::RS) & 1u) ^ 1u, lim,
                           abort_flag))
              break;
            const uint32_t rb = smem_u32(&rsa_full[rs]);
            mbar_arrive_expect_tx(rb, C::RSA);
            tma_load_2d(smem_u32(rsa + rs * (C::RSA / 2)), &tmSA, rb, g0 + i, m0);
            last_sa = b;
          }
          // weight-scale blocks start on even steps (multiples of 8 weight groups)
          if (sw_tma && (i == 0 || wblock(i) != wblock(i - 1))) {
            const int b = wblock(i) - wblock(0), rw = b % C::RW;
            if (!mbar_wait(smem_u32(&rsw_empty[rw]), ((uint32_t)(b / C::RW) & 1u) ^ 1u, lim,
                           abort_flag))
              break;
            const uint32_t wb = smem_u32(&rsw_full[rw]);
            mbar_arrive_expect_tx(wb, C::RSW);
            tma_load_2d(smem_u32(rsw + rw * (C::RSW / 2)), &tmSW, wb, wblock(i) * 8, n0);
            last_sw = b;
          }
        }
        const uint32_t fb = smem_u32(&pk_full[st]);
        mbar_arrive_expect_tx(fb, C::PK_STAGE);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE), &tmW, fb, (g0 + i) * 64, n0);
        tma_load_2d(smem_u32(pk + st * C::PK_STAGE + C::PKW), &tmA, fb, (g0 + i) * 64, m0);
        trace_stamp(args, 0, sidx);
        last = sidx;
      }
      // Never leave the CTA with bulk copies in flight: wait for the last stages issued.
      for (int i = (last - C::NP + 1 > 0 ? last - C::NP + 1 : 0); i <= last; ++i) {
        if (i == args.withhold) continue;
        mbar_wait(smem_u32(&pk_full[i % C::NP]), (uint32_t)(i / C::NP) & 1u, lim, never);
      }
      for (int b = (last_sa - C::RS + 1 > 0 ? last_sa - C::RS + 1 : 0); b <= last_sa; ++b)
        mbar_wait(smem_u32(&rsa_full[b % C::RS]), (uint32_t)(b / C::RS) & 1u, lim, never);
      for (int b = (last_sw - C::RW + 1 > 0 ? last_sw - C::RW + 1 : 0); b <= last_sw; ++b)
        mbar_wait(smem_u32(&rsw_full[b % C::RW]), (uint32_t)(b / C::RW) & 1u, lim, never);
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
    const int ns = (ng + C::KPS - 1) / C::KPS;
    for (int sidx = 0; sidx < ns; ++sidx) {
      const int st = sidx % C::NP;
      const int i0 = sidx * C::KPS;
      const int nk = min(C::KPS, ng - i0);   // groups of this stage inside the split
      bool ok = mbar_wait(smem_u32(&pk_full[st]), (uint32_t)(sidx / C::NP) & 1u, lim, abort_flag);
      for (int j = 0; j < nk; ++j)
        ok = ok && mbar_wait(smem_u32(&x_empty[(i0 + j) % C::NX]),
                             ((uint32_t)((i0 + j) / C::NX) & 1u) ^ 1u, lim, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const uint8_t* pw = pk + st * C::PK_STAGE;
      const uint8_t* pa = pw + C::PKW;
#pragma unroll
      for (int j = 0; j < C::KPS; ++j) {
        if (j < nk) {
          const int xs = (i0 + j) % C::NX;
          // weight row -> tensor memory (16-byte chunk c of a row sits at c ^ (row & 7))
          uint32_t wv[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(
                pw + row * 128 + (((4 * j + c) ^ (row & 7)) << 4));
            wv[4 * c + 0] = v.x;
            wv[4 * c + 1] = v.y;
            wv[4 * c + 2] = v.z;
            wv[4 * c + 3] = v.w;
          }
          uint32_t e0[16], e1[16];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            e0[2 * q] = expand_lo(wv[q]);
            e0[2 * q + 1] = expand_hi(wv[q]);
            e1[2 * q] = expand_lo(wv[8 + q]);
            e1[2 * q + 1] = expand_hi(wv[8 + q]);
          }
          const uint32_t tw = tbase + t_lane + C::W_COL0 + xs * 32;
          tmem_st16(tw, e0);
          tmem_st16(tw + 16, e1);
          // token rows -> shared memory, 128-byte-swizzled K-major operand layout
          uint8_t* xd = xa + xs * C::XA;
#pragma unroll
          for (int it = ct; it < BT * 8; it += 128) {
            const int r = it >> 3, u = it & 7;
            const uint2 v = *reinterpret_cast<const uint2*>(
                pa + r * 128 + (((4 * j + (u >> 1)) ^ (r & 7)) << 4) + ((u & 1) << 3));
            uint4 o;
            o.x = expand_lo(v.x);
            o.y = expand_hi(v.x);
            o.z = expand_lo(v.y);
            o.w = expand_hi(v.y);
            *reinterpret_cast<uint4*>(xd + r * 128 + ((u ^ (r & 7)) << 4)) = o;
          }
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
      if (threadIdx.x == 32 * C::CONV0) trace_stamp(args, 1, sidx);
    }
  } else if (warp == C::LOADER && SCT && !DUMP) {
    // ------------------------------------------------------------ scale loader (TMA path)
    // Raw blocks [rows][8 groups] fp16 -> per-group fp32 slots sa[BT] | sw[BM]*2^-8.
    constexpr int NA = (BT + 31) / 32;
    float swc[4];   // per-row weight scale when K/gw == 1
    if (!sw_tma) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + lane + 32 * j;
        swc[j] = n < args.N ? __half2float(args.sw[(size_t)n * args.Gw]) * (1.0f / 256.0f) : 0.0f;
      }
    }
    bool ok = true;
    int cur_w = -1;   // raw sw block currently held
    for (int i = 0; i < ng && ok; ++i) {
      const int b = i >> 3;
      if ((i & 7) == 0) {
        ok = mbar_wait(smem_u32(&rsa_full[b % C::RS]), (uint32_t)(b / C::RS) & 1u, lim, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if (sw_tma && wblock(i) - wblock(0) != cur_w) {
        __syncwarp();
        if (cur_w >= 0 && lane == 0) mbar_arrive(smem_u32(&rsw_empty[cur_w % C::RW]));
        cur_w = wblock(i) - wblock(0);
        ok = mbar_wait(smem_u32(&rsw_full[cur_w % C::RW]), (uint32_t)(cur_w / C::RW) & 1u, lim,
                       abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      ok = mbar_wait(smem_u32(&sc_empty[i % C::SR]), ((uint32_t)(i / C::SR) & 1u) ^ 1u, lim,
                     abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      float* slot = s_sc + (i % C::SR) * (BT + C::BM);
      const uint16_t* ra = rsa + (b % C::RS) * (C::RSA / 2) + (i & 7);
#pragma unroll
      for (int j = 0; j < NA; ++j) {
        const int t = lane + 32 * j;
        if (t < BT) slot[t] = __half2float(__ushort_as_half(ra[t * 8]));
      }
      if (sw_tma) {
        const int wj = ((g0 + i) * 128 / args.gw) & 7;
        const uint16_t* rw = rsw + (cur_w % C::RW) * (C::RSW / 2) + wj;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          slot[BT + lane + 32 * j] =
              __half2float(__ushort_as_half(rw[(lane + 32 * j) * 8])) * (1.0f / 256.0f);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) slot[BT + lane + 32 * j] = swc[j];
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&sc_full[i % C::SR]));
        trace_stamp(args, 4, i);
        if ((i & 7) == 7 || i == ng - 1) mbar_arrive(smem_u32(&rsa_empty[b % C::RS]));
      }
    }
    __syncwarp();
    if (ok && cur_w >= 0 && lane == 0) mbar_arrive(smem_u32(&rsw_empty[cur_w % C::RW]));
  } else if (warp == C::LOADER) {
    // ------------------------------------------------------------ scale loader (generic)
    // Groups are loaded in batches of SB so that SB groups' global loads are in flight
    // together; each slot holds fp32 sa[BT] (tokens m0..) and sw[BM] * 2^-8 (weight rows).
    constexpr int NA = (BT + 31) / 32;
    for (int i0 = 0; i0 < ng; i0 += C::SB) {
      const int nb = min(C::SB, ng - i0);
      bool ok = true;
      for (int b = 0; b < nb; ++b)
        ok = ok && mbar_wait(smem_u32(&sc_empty[(i0 + b) % C::SR]),
                             ((uint32_t)((i0 + b) / C::SR) & 1u) ^ 1u, lim, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      float va[C::SB][NA], vw[C::SB][4];
#pragma unroll
      for (int b = 0; b < C::SB; ++b) {
        const int g = g0 + i0 + b;
        const bool live = b < nb && !DUMP;
#pragma unroll
        for (int j = 0; j < NA; ++j) {
          const int t = lane + 32 * j;
          const int m = m0 + t;
          va[b][j] = (live && t < BT && m < args.M)
                         ? __half2float(args.sa[(size_t)m * args.G + g]) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n = n0 + lane + 32 * j;
          vw[b][j] = (live && n < args.N)
                         ? __half2float(args.sw[(size_t)n * args.Gw + (g * 128) / args.gw]) *
                               (1.0f / 256.0f)
                         : 0.0f;
        }
      }
#pragma unroll
      for (int b = 0; b < C::SB; ++b) {
        if (b < nb) {
          float* slot = s_sc + ((i0 + b) % C::SR) * (BT + C::BM);
#pragma unroll
          for (int j = 0; j < NA; ++j)
            if (lane + 32 * j < BT) slot[lane + 32 * j] = va[b][j];
#pragma unroll
          for (int j = 0; j < 4; ++j) slot[BT + lane + 32 * j] = vw[b][j];
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sc_full[(i0 + b) % C::SR]));
          if (lane == 0) trace_stamp(args, 4, i0 + b);
        }
      }
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
    // One weight group spans this CTA's whole K-range: sw factors out of the sum.
    const bool hoist = (g0 * 128) / args.gw == ((g0 + ng - 1) * 128) / args.gw;

    float2 acc[C::CPT / 2];
#pragma unroll
    for (int e = 0; e < C::CPT / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
    float sw_hoisted = 0.0f;

    bool ok = true;
    for (int i = 0; i < ng; ++i) {
      const int g = g0 + i;
      const int sl = i % C::NSLOT;
      const int sc = i % C::SR;
      ok = mbar_wait(smem_u32(&d_full[sl]), (uint32_t)(i / C::NSLOT) & 1u, lim, abort_flag);
      ok = ok && mbar_wait(smem_u32(&sc_full[sc]), (uint32_t)(i / C::SR) & 1u, lim, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float* slot = s_sc + sc * (BT + C::BM);
      const float swv = slot[BT + row];
      if (i == 0) sw_hoisted = swv;
      const float2 sw2 = make_float2(swv, swv);
      const float4* sab = reinterpret_cast<const float4*>(slot + h * 64);
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
        mbar_arrive(smem_u32(&sc_empty[sc]));
      }
      if (et == 0) trace_stamp(args, 3, i);
    }
    const bool aborted = bar_red_or(1, NE, !ok);

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
