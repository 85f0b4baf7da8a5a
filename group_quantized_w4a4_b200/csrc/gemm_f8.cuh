// gemm_f8.cuh -- the W4A4 GEMM for compute-bound shapes (many tokens), with the 4-bit
// values carried as E4M3 codes so that the tensor core returns every group's exact integer
// partial already in fp32.
//
// The method ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing",
// abstract) multiplies 4-bit integers on the tensor cores and dequantises each 128-wide
// K-group's integer partial on the CUDA cores:
//   Y[m,n] = sum_g P_g[m,n] * sa[m,g] * sw[n, g*128/gw],  P_g = sum_{k in g} qa[m,k]*qw[n,k].
// On B200 the per-group dequantisation, not the MMA, limits this (the abstract's "group
// dequantization overhead" on the CUDA cores; B200's tensor : CUDA-core throughput ratio is
// A100-like).  An int8 MMA leaves an int32 partial that costs an int->fp32 conversion per
// partial on top of the scale arithmetic.  Every q in [-8, 7] is an E4M3 value, and so is
// every product (|qa*qw| <= 64); a group's sum of 128 such products is an integer of at most
// 2^13 in magnitude, which the fp32 accumulator of kind::f8f6f4 holds exactly.  So with the
// operands stored as E4M3 codes of q (one byte per element, written by the quantizer), the
// MMA gives the same exact P_g as an int8 MMA, as an fp32 value, and the epilogue only
// multiplies and adds.  (Exactness is checked bit for bit against the oracle's int64
// partials by the partials export of this kernel.)
//
// Tile: 128 tokens (tensor-memory lanes, MMA M) x 256 weight rows (MMA N), one K-group per
// pipeline stage: a [128 x 128 B] token box and a [256 x 128 B] weight box, both by TMA with
// 128-byte swizzle into a 4-deep ring.  Per K-group, 4 MMAs (K = 32 each) write the group's
// partial into one of two 256-column tensor-memory slots, so the epilogue drains one slot
// while the next group's MMAs fill the other.
// Roles (384 threads in three warpgroups, one persistent CTA per SM, whole tiles
// round-robin):
//   warp 0       TMA producer (lane 0 issues)
//   warp 1       MMA issuer (lane 0 issues; commits free the stage and fill the slot)
//   warps 2, 3   idle (they only complete the first warpgroup)
//   warps 4..11  epilogue: warp w reads tensor-memory lanes 32*(w%4)..+31 (one token each)
//                and columns 128*((w-4)/4)..+127 of the slot; per group and column:
//                s = sa*sw (fp32, exact), acc += P*s (packed f32x2 math).
// The block launches with 168 registers a thread (three warps per SM sub-partition); the
// first warpgroup then gives up all but 40 and the two epilogue warpgroups take 232, which
// their 128 accumulators and two 32-column partial loads in flight need.
// Weight scales are staged in shared memory as fp32 [8 groups][256 columns] per block of 8
// K-groups, two blocks (the next one is loaded while the current one is used); each
// epilogue thread keeps its token's scales in registers, also one block ahead.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "quantize.cuh"

namespace apex {

// Epilogue modes: per-group weight scales (any weight group), one weight scale per row for
// the whole K (per-channel weight groups: the scale is applied once, after the sum), or the
// partials export.
enum F8Mode : int { F8_GROUPED = 0, F8_PER_CHANNEL = 1, F8_DUMP = 2 };

struct F8Args {
  int M, N, K;
  int G;             // K / 128
  int Gw;            // K / gw
  int gpg;           // K-groups per weight scale (gw / 128)
  int gpg_shift;     // log2(gpg) when gpg is a power of two, else -1
  int tiles_m, tiles_n, T;
  int P;             // persistent CTAs (gridDim.x)
  int sa_vec;        // sa rows readable as 16-byte blocks of 8 groups
  int sw_vec;        // sw rows readable as 16-byte blocks of 8 groups (gw == 128)
  int y_vec;         // Y rows writable as 16-byte vectors
  const __half* sa;  // [M][G]
  const __half* sw;  // [N][Gw]
  __half* y;         // [M][N]
  int32_t* dump;     // [G][M][N] per-group partials (export kernel only)
  unsigned long long wait_ns;
  // Optional quantized output (QOUT instantiations): Y's fp16 values quantized as the next
  // layer's activations, E4M3 codes [M][N] and fp16 scales [M][N/128].  y may then be null.
  uint8_t* qout;
  __half* qscale;
  // The outlier dual path (0: none): NO extra K-steps of 64 fp16 channels per tile, from the
  // maps tmXo (x_out [M][64*NO]) and tmWo (w_out [N][64*NO]), multiplied by kind::f16 MMAs
  // and added with unit scale after the 4-bit groups.
  int NO;
};

// EW: epilogue warps, 8 (128 columns a thread, 32-column partial loads double-buffered) or
// 16 (64 columns a thread, twice the warps to cover latencies, 16-column loads).
template <int EW>
struct F8Cfg {
  static constexpr int BM = 128;                   // tokens per tile
  static constexpr int BN = 256;                   // weight rows per tile
  static constexpr int NS = 4;                     // operand stages, one K-group each
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;  // 48 KB
  static constexpr int SLOTS = 2;                  // partial slots of BN columns
  static constexpr int TMEM_COLS = SLOTS * BN;     // 512
  static constexpr int EPI_WARPS = EW;
  static constexpr int EPI_THREADS = EW * 32;
  static constexpr int THREADS = 128 + EPI_THREADS;
  // registers: what __launch_bounds__(THREADS, 1) allows (warps per SM sub-partition x 32 x
  // registers <= 16384), then the first warpgroup keeps REGS_CTRL and the epilogue takes
  // REGS_EPI
  static constexpr int REGS_LAUNCH = EW == 8 ? 168 : 96;
  static constexpr int REGS_CTRL = EW == 8 ? 40 : 24;
  static constexpr int REGS_EPI = EW == 8 ? 232 : 112;
  static_assert(128 * REGS_CTRL + EPI_THREADS * REGS_EPI <= THREADS * REGS_LAUNCH,
                "register budgets fit the block's pool");
  static constexpr int CPT = BN * 4 / EW;          // columns per epilogue thread
  static constexpr int LC = EW == 8 ? 32 : 16;     // columns per tensor-memory load
  static constexpr bool DBUF = EW == 8;            // next load in flight during the current
  static constexpr int SPT = 8 * BN / EPI_THREADS;  // staged weight scales per thread
  static constexpr int SWB = 8 * BN * 2;           // one staged block of weight scales (fp16)
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_SW = NS * STAGE;
  static constexpr int OFF_BAR = OFF_SW + 2 * SWB;
  static constexpr int NBAR = 2 * NS + 2 * SLOTS + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;   // + alignment slack
  static_assert(STAGE % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(TMEM_COLS <= 512, "tensor memory budget");
  static_assert(CPT % LC == 0 && (SPT == 8 || SPT == 4), "epilogue split");
};

// Tile t -> (token tile, weight tile), token tiles fastest: the CTAs running at once cover all
// token tiles of a few weight tiles, so each weight tile streams from HBM about once and is
// read by every token tile while it is in L2 (the activations, a few tens of MB, stay in L2).
__device__ __forceinline__ void f8_tile(const F8Args& a, int t, int& tm, int& tn) {
  tm = t % a.tiles_m;
  tn = t / a.tiles_m;
}

// The NG (8 or 4) fp16 scales of groups g0 .. g0+NG-1 of one row (raw bits, packed two per
// 32-bit word; zeros outside [0, G) and for rows outside the matrix): one 16- or 8-byte load
// when `vec` (consecutive scale groups, aligned), else one load per group; gpg = K-groups per
// scale group.
template <int NG>
__device__ __forceinline__ uint4 scale_block(const __half* base, int row, int rows, int ld,
                                             int g0, int G, int gpg, bool vec,
                                             int gpg_shift = 0) {
  if (row >= rows) return make_uint4(0, 0, 0, 0);
  const __half* r = base + (size_t)row * ld;
  if (vec) {
    if constexpr (NG == 8) return __ldg(reinterpret_cast<const uint4*>(r + g0));
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(r + g0));
    return make_uint4(v.x, v.y, 0u, 0u);
  }
  uint32_t h[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  if (gpg_shift >= 0) {   // coarse groups: repeated indices, which the loads share
#pragma unroll
    for (int j = 0; j < NG; ++j)
      h[j] = g0 + j < G ? (uint32_t)__half_as_ushort(__ldg(r + ((g0 + j) >> gpg_shift))) : 0u;
  } else {
#pragma unroll
    for (int j = 0; j < NG; ++j)
      h[j] = g0 + j < G ? (uint32_t)__half_as_ushort(r[(g0 + j) / gpg]) : 0u;
  }
  return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                    h[6] | (h[7] << 16));
}

__device__ __forceinline__ uint16_t half_bits_at(const uint4& v, int j) {
  const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
  return (uint16_t)((j & 1) ? (w >> 16) : (w & 0xFFFFu));
}

// (sa * sw_lo, sa * sw_hi) in fp32 from fp16 bits: one mixed-precision fma each (f16 inputs,
// f32 result, + 0), exact, since the product of two fp16 values fits fp32's significand and
// range.
__device__ __forceinline__ float2 scale_pair(uint32_t sw2, uint16_t sa) {
  float lo, hi;
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "fma.rn.f32.f16 %0, %3, l, 0f00000000;\n\t"
      "fma.rn.f32.f16 %1, %3, h, 0f00000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(sw2), "h"(sa));
  return make_float2(lo, hi);
}

__device__ __forceinline__ float half_at(const uint4& v, int j) {
  const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
  return __half2float(__ushort_as_half((uint16_t)((j & 1) ? (w >> 16) : (w & 0xFFFFu))));
}

__device__ __forceinline__ uint32_t half2_bits(float2 v) {
  const __half2 h = __float22half2_rn(v);
  return *reinterpret_cast<const uint32_t*>(&h);
}


// DUAL: the outlier dual path's K-steps are compiled in (args.NO of them; else none).
// QOUT: the output is also quantized as the next layer's E4M3-coded activations.
template <int MODE, int EW, bool DUAL = false, bool QOUT = false>
__global__ void __launch_bounds__(F8Cfg<EW>::THREADS, 1)
    w4a4_gemm_f8_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmXo,
                        const __grid_constant__ CUtensorMap tmWo, const F8Args args) {
  using C = F8Cfg<EW>;
  constexpr bool DUMP = MODE == F8_DUMP;
  constexpr bool PERCH = MODE == F8_PER_CHANNEL;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem + C::OFF_STAGE;
  uint16_t* s_sw = reinterpret_cast<uint16_t*>(smem + C::OFF_SW);   // fp16 bits
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                 // stage loaded (TMA bytes)
  uint64_t* empty = full + C::NS;        // stage read by its MMAs (commit)
  uint64_t* tfull = empty + C::NS;       // slot holds a finished partial (commit)
  uint64_t* tempty = tfull + C::SLOTS;   // slot read out (one arrival per epilogue warp)
  uint64_t* mma_done = tempty + C::SLOTS;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* s_abort = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* s_never = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = args.wait_ns;
  const int G = args.G;
  const int NO = DUAL ? args.NO : 0;
  const int GT = args.G + NO;        // K-steps per tile: the 4-bit groups, then the outliers

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
    }
    for (int i = 0; i < C::SLOTS; ++i) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), C::EPI_WARPS);
    }
    mbar_init(smem_u32(mma_done), 1);
    *s_abort = 0;
    *s_never = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (NO > 0) {
      tma_prefetch_desc(&tmXo);
      tma_prefetch_desc(&tmWo);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched as a programmatic dependent: the prologue above overlaps the previous grid's
  // tail; the roles that touch global memory wait for it below
  grid_dep_launch();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(s_tmem);
  volatile int* abort_flag = s_abort;
  volatile int* never = s_never;
  // Role dispatch by warpgroup first, so that each register budget covers exactly the code
  // of its warpgroup.
  if (warp < 4) {
    regs_dec<C::REGS_CTRL>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    grid_dep_wait();
    int it = 0, last = -1;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < args.T; t += args.P) {
      int tm, tn;
      f8_tile(args, t, tm, tn);
      for (int g = 0; g < GT; ++g, ++it) {
        const int st = it % C::NS;
        ok = mbar_wait(smem_u32(&empty[st]), ((uint32_t)(it / C::NS) & 1u) ^ 1u, lim, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          const uint32_t fb = smem_u32(&full[st]);
          uint8_t* sa_dst = stages + st * C::STAGE;
          mbar_arrive_expect_tx(fb, C::STAGE);
          if (g < G) {   // 128 E4M3 codes of each row: one K-group
            tma_load_2d(smem_u32(sa_dst), &tmA, fb, g * 128, tm * C::BM);
            tma_load_2d(smem_u32(sa_dst + C::A_BYTES), &tmB, fb, g * 128, tn * C::BN);
          } else {       // 64 fp16 outlier channels of each row (the same 128 bytes a row)
            tma_load_2d(smem_u32(sa_dst), &tmXo, fb, (g - G) * 64, tm * C::BM);
            tma_load_2d(smem_u32(sa_dst + C::A_BYTES), &tmWo, fb, (g - G) * 64, tn * C::BN);
          }
        }
        __syncwarp();
        last = it;
      }
    }
    // never leave the CTA with bulk copies in flight
    for (int s = (last - C::NS + 1 > 0 ? last - C::NS + 1 : 0); s <= last; ++s)
      mbar_wait(smem_u32(&full[s % C::NS]), (uint32_t)(s / C::NS) & 1u, lim, never);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_e4m3(C::BM, C::BN);
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < args.T; t += args.P) {
      for (int g = 0; g < GT; ++g, ++it) {
        const int st = it % C::NS, sl = it % C::SLOTS;
        ok = mbar_wait2(smem_u32(&full[st]), (uint32_t)(it / C::NS) & 1u,
                        smem_u32(&tempty[sl]), ((uint32_t)(it / C::SLOTS) & 1u) ^ 1u, lim,
                        abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          const uint64_t a0 = smem_desc_k_sw128(smem_u32(stages + st * C::STAGE));
          const uint64_t b0 = smem_desc_k_sw128(smem_u32(stages + st * C::STAGE + C::A_BYTES));
          const uint32_t d = tbase + sl * C::BN;
          // 32 bytes of K per MMA (+2 in 16-byte descriptor units): 32 E4M3 codes, or 16 fp16
          // outlier channels (kind::f16; the descriptor's type fields read the same)
          if (g < G) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_f8_ss(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc, j > 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              umma_f16_ss(d, a0 + (uint64_t)(2 * j), b0 + (uint64_t)(2 * j), idesc,
                          j > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&empty[st]));
          umma_commit(smem_u32(&tfull[sl]));
        }
        __syncwarp();
      }
    }
    if (lane == 0) umma_commit(smem_u32(mma_done));
    __syncwarp();
    mbar_wait(smem_u32(mma_done), 0u, lim, never);
    __syncwarp();
  }
  } else {
    regs_inc<C::REGS_EPI>();
    // ------------------------------------------------------------ epilogue
    grid_dep_wait();   // scales and outputs are global memory
    const int ew = warp - 4;                    // 0 .. EW-1
    const int et = threadIdx.x - 128;           // stages weight column et % 256
    const int lq = warp & 3;                    // tensor-memory lane quarter of this warp
    const int ch = ew >> 2;                     // columns CPT*ch .. +CPT-1
    const int row = 32 * lq + lane;             // token of the tile
    const uint32_t t_lane = (uint32_t)(32 * lq) << 16;
    constexpr uint32_t EB = 1;                  // named barrier of the epilogue warps
    const bool sa_vec = args.sa_vec != 0, sw_vec = args.sw_vec != 0;
    float2 acc[C::CPT / 2];
    bool ok = true, aborted = false;
    int it = 0;
    int b = 0;   // flat 8-group block counter: its weight scales are staged in s_sw[b & 1]

    // weight scales of one block, as fp16 bits: thread et stages column et % 256, groups
    // SPT*(et / 256) .. +SPT-1
    const int sw_col = et & 255, sw_g0 = C::SPT * (et >> 8);
    // (per-channel weight groups: only the column's one scale, in group row 0)
    auto stage_sw = [&](uint16_t* blk, const uint4& v) {
      if constexpr (PERCH) {
        if (sw_g0 == 0) blk[sw_col] = (uint16_t)(v.x & 0xFFFFu);
      } else {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < C::SPT; ++j)
          blk[(sw_g0 + j) * C::BN + sw_col] =
              (uint16_t)((j & 1) ? (w[j / 2] >> 16) : (w[j / 2] & 0xFFFFu));
      }
    };
    auto load_sw = [&](int tn, int gb8) {
      if constexpr (PERCH) {
        const int n = tn * C::BN + sw_col;
        return make_uint4(sw_g0 == 0 && n < args.N ? __half_as_ushort(args.sw[n]) : 0u, 0u, 0u,
                          0u);
      } else {
        return scale_block<C::SPT>(args.sw, tn * C::BN + sw_col, args.N, args.Gw, gb8 + sw_g0,
                                   G, args.gpg, sw_vec, args.gpg_shift);
      }
    };
    // the first block's scales before the first group
    int t = blockIdx.x;
    uint4 sa_c = make_uint4(0, 0, 0, 0);
    if (t < args.T && !DUMP) {
      int tm, tn;
      f8_tile(args, t, tm, tn);
      stage_sw(s_sw, load_sw(tn, 0));
      sa_c = scale_block<8>(args.sa, tm * C::BM + row, args.M, G, 0, G, 1, sa_vec);
    }
    aborted = bar_red_or(EB, C::EPI_THREADS, false);
    for (; !aborted && t < args.T; t += args.P) {
      int tm, tn;
      f8_tile(args, t, tm, tn);
      const int m = tm * C::BM + row;
      const int n0 = tn * C::BN + ch * C::CPT;
#pragma unroll
      for (int e = 0; e < C::CPT / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
      for (int gb8 = 0; gb8 < G; gb8 += 8, ++b) {
        // the next block's scales (of this tile, or the first of the next) are in flight
        // while this block is processed
        const bool more = gb8 + 8 < G;
        int ntm = tm, ntn = tn;
        if (!more && t + args.P < args.T) f8_tile(args, t + args.P, ntm, ntn);
        const bool have_next = !DUMP && (more || t + args.P < args.T);
        const int ngb = more ? gb8 + 8 : 0;
        uint4 sw_n = make_uint4(0, 0, 0, 0), sa_n = make_uint4(0, 0, 0, 0);
        if (have_next) {
          sw_n = load_sw(ntn, ngb);
          sa_n = scale_block<8>(args.sa, ntm * C::BM + row, args.M, G, ngb, G, 1, sa_vec);
        }
        const uint16_t* swb = s_sw + (b & 1) * (C::SWB / 2) + ch * C::CPT;
        const int je = min(8, G - gb8);
        for (int j = 0; j < je && ok; ++j, ++it) {
          const int sl = it % C::SLOTS;
          ok = mbar_wait(smem_u32(&tfull[sl]), (uint32_t)(it / C::SLOTS) & 1u, lim, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint32_t td = tbase + t_lane + sl * C::BN + ch * C::CPT;
          const uint16_t sa_h = half_bits_at(sa_c, j);
          const float saf = __half2float(__ushort_as_half(sa_h));
          const float2 sa2 = make_float2(saf, saf);
          const uint16_t* swj = swb + j * C::BN;
          // NCH loads of LC columns; with DBUF the next one is in flight while the current
          // one is used
          constexpr int NCH = C::CPT / C::LC;
          uint32_t p[C::DBUF ? 2 : 1][C::LC];
          auto ld = [&](int cc, uint32_t* dst) {
            if constexpr (C::LC == 32) tmem_ld32_nowait(td + 32 * cc, dst);
            else tmem_ld16_nowait(td + 16 * cc, dst);
          };
          auto ld_wait = [&](uint32_t* dst) {
            if constexpr (C::LC == 32) tmem_ld_wait32(dst);
            else tmem_ld_wait16(dst);
          };
          auto release = [&]() {   // every load of the slot has completed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&tempty[sl]));
          };
          if constexpr (C::DBUF) {
            ld(0, p[0]);
            ld_wait(p[0]);
          }
#pragma unroll
          for (int cc = 0; cc < NCH; ++cc) {
            uint32_t* pc = p[C::DBUF ? (cc & 1) : 0];
            if constexpr (C::DBUF) {
              if (cc + 1 < NCH) ld(cc + 1, p[(cc + 1) & 1]);
            } else {
              ld(cc, pc);
              ld_wait(pc);
              if (cc == NCH - 1) release();
            }
            if constexpr (DUMP) {
              int32_t* dst =
                  args.dump + ((size_t)(gb8 + j) * args.M + m) * args.N + n0 + cc * C::LC;
#pragma unroll
              for (int e = 0; e < C::LC; ++e)
                if (m < args.M && n0 + cc * C::LC + e < args.N)
                  dst[e] = __float2int_rn(__uint_as_float(pc[e]));
            } else if constexpr (PERCH) {
              // one weight scale for all of K: acc += P * sa here, times sw after the sum
#pragma unroll
              for (int q = 0; q < C::LC / 2; ++q)
                acc[cc * (C::LC / 2) + q] = __ffma2_rn(
                    make_float2(__uint_as_float(pc[2 * q]), __uint_as_float(pc[2 * q + 1])), sa2,
                    acc[cc * (C::LC / 2) + q]);
            } else {
              // s = sa * sw, exact in fp32, from the fp16 scales in one mixed-precision fma
#pragma unroll
              for (int q = 0; q < C::LC / 8; ++q) {
                const uint4 w8 = *reinterpret_cast<const uint4*>(swj + cc * C::LC + 8 * q);
                const uint32_t w[4] = {w8.x, w8.y, w8.z, w8.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const int e = cc * (C::LC / 2) + 4 * q + h;
                  acc[e] = __ffma2_rn(make_float2(__uint_as_float(pc[8 * q + 2 * h]),
                                                  __uint_as_float(pc[8 * q + 2 * h + 1])),
                                      scale_pair(w[h], sa_h), acc[e]);
                }
              }
            }
            if constexpr (C::DBUF) {
              if (cc + 1 < NCH) ld_wait(p[(cc + 1) & 1]);
              if (cc == NCH - 2) release();
            }
          }
        }
        // the next block's weight scales into the other buffer; one barrier per block (also
        // the epilogue's one decision to give up, so no warp is left waiting here)
        if (have_next) stage_sw(s_sw + ((b + 1) & 1) * (C::SWB / 2), sw_n);
        aborted = bar_red_or(EB, C::EPI_THREADS, !ok);
        if (aborted) break;
        sa_c = sa_n;
      }
      if (aborted) break;
      if constexpr (PERCH) {
        // the row's one weight scale, applied to the finished sum of the 4-bit groups: it was
        // staged with the tile's last block (every group row of the block holds it)
        const uint16_t* swl = s_sw + ((b - 1) & 1) * (C::SWB / 2) + ch * C::CPT;
#pragma unroll
        for (int e8 = 0; e8 < C::CPT; e8 += 8) {
          const uint4 w8 = *reinterpret_cast<const uint4*>(swl + e8);
          const uint32_t w[4] = {w8.x, w8.y, w8.z, w8.w};
#pragma unroll
          for (int h = 0; h < 4; ++h)
            acc[e8 / 2 + h] = __fmul2_rn(acc[e8 / 2 + h],
                                         make_float2(__half2float(__ushort_as_half((uint16_t)(w[h] & 0xFFFFu))),
                                                     __half2float(__ushort_as_half((uint16_t)(w[h] >> 16)))));
        }
      }
      if constexpr (!DUMP) {
        // the outlier channels' 16-bit products, added with unit scale; a wait that gives up
        // leaves the rest to the next block barrier (no warp can be left behind there)
        for (int o = 0; o < NO && ok; ++o, ++it) {
          const int sl = it % C::SLOTS;
          ok = mbar_wait(smem_u32(&tfull[sl]), (uint32_t)(it / C::SLOTS) & 1u, lim, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const uint32_t td = tbase + t_lane + sl * C::BN + ch * C::CPT;
#pragma unroll
          for (int cc = 0; cc < C::CPT / C::LC; ++cc) {
            uint32_t p[C::LC];
            if constexpr (C::LC == 32) {
              tmem_ld32_nowait(td + 32 * cc, p);
              tmem_ld_wait32(p);
            } else {
              tmem_ld16_nowait(td + 16 * cc, p);
              tmem_ld_wait16(p);
            }
            if (cc == C::CPT / C::LC - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&tempty[sl]));
            }
#pragma unroll
            for (int q = 0; q < C::LC / 2; ++q)   // P * 1 + acc: one rounding, as an add
              acc[cc * (C::LC / 2) + q] = __ffma2_rn(
                  make_float2(__uint_as_float(p[2 * q]), __uint_as_float(p[2 * q + 1])),
                  make_float2(1.0f, 1.0f), acc[cc * (C::LC / 2) + q]);
          }
        }
        // the finished tile: this thread's token row, 128 consecutive outputs (after a wait
        // that gave up, nothing: the next block barrier takes the decision to stop)
        if (ok && m < args.M && args.y != nullptr) {
          __half* dst = args.y + (size_t)m * args.N + n0;
          if (args.y_vec && n0 + C::CPT <= args.N) {
#pragma unroll
            for (int e = 0; e < C::CPT / 2; e += 4)
              *reinterpret_cast<uint4*>(dst + 2 * e) =
                  make_uint4(half2_bits(acc[e]), half2_bits(acc[e + 1]), half2_bits(acc[e + 2]),
                             half2_bits(acc[e + 3]));
          } else {
#pragma unroll
            for (int e = 0; e < C::CPT; ++e) {
              const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
              if (n0 + e < args.N) dst[e] = __float2half_rn(v);
            }
          }
        }
        if constexpr (QOUT) {
          // The next layer's activations: this thread's 128 outputs of token m are exactly one
          // 128-wide K-group of that token's input to the next layer (N % 128 == 0), so the
          // group's scale and E4M3 codes are made here, from the fp16 values Y holds and with
          // the activation quantizer's own rule; no other thread is involved.  (A tile's
          // upper half may lie past N: N % 128 == 0, so n0 < N means all 128 are inside.)
          if (ok && m < args.M && n0 < args.N) {
            float amax = 0.0f;
#pragma unroll
            for (int e = 0; e < C::CPT / 2; ++e)
              amax = fmaxf(amax, fmaxf(fabsf(acc[e].x), fabsf(acc[e].y)));
            // rounding to fp16 is monotonic: the largest |fp16(v)| is fp16(largest |v|)
            const __half sc = group_scale(__half2float(__float2half_rn(amax)));
            const QScale qs = make_qscale(__half2float(sc));
            uint8_t* qd = args.qout + (size_t)m * args.N + n0;
#pragma unroll
            for (int e = 0; e < C::CPT / 2; e += 8) {
              const uint4 h0 = make_uint4(half2_bits(acc[e]), half2_bits(acc[e + 1]),
                                          half2_bits(acc[e + 2]), half2_bits(acc[e + 3]));
              const uint4 h1 = make_uint4(half2_bits(acc[e + 4]), half2_bits(acc[e + 5]),
                                          half2_bits(acc[e + 6]), half2_bits(acc[e + 7]));
              const uint2 c0 = quant_e4m3_8(h0, qs), c1 = quant_e4m3_8(h1, qs);
              *reinterpret_cast<uint4*>(qd + 2 * e) = make_uint4(c0.x, c0.y, c1.x, c1.y);
            }
            args.qscale[(size_t)m * (args.N / 128) + n0 / 128] = sc;
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

// Packed int4 [rows][K/2] -> E4M3 codes of the same q [rows][K] (element order): each thread
// turns 8 packed bytes into 16 codes (e4m3_of_nibbles, quantize.cuh).
__global__ void __launch_bounds__(256) unpack_e4m3_kernel(const uint8_t* __restrict__ packed,
                                                         int64_t words, uint8_t* __restrict__ codes) {
  grid_dep_wait();
  grid_dep_launch();
  // one unit = 8 packed bytes (16 elements) -> 16 codes
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(packed) + i);
    uint4 o;
    o.x = e4m3_of_nibbles(w.x);
    o.y = e4m3_of_nibbles(w.x >> 16);
    o.z = e4m3_of_nibbles(w.y);
    o.w = e4m3_of_nibbles(w.y >> 16);
    reinterpret_cast<uint4*>(codes)[i] = o;
  }
}

}  // namespace apex
