// gemm.cuh -- W4A4 group-quantized GEMM on sm_100a tensor cores (tcgen05, kind::i8).
//
// Computes Y[m,n] = sum_g P_g[m,n] * sa[m,g] * sw[n, g*128/gw], where
// P_g = sum over the 128-wide K-group g of qa[m,k]*qw[n,k] is an exact integer
// ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute Rebalancing", abstract:
// INT4 tensor-core products with per-group dequantisation on the CUDA cores; the
// mixed-granularity mode keeps 128-wide activation groups and coarser weight groups).
//
// Tile: 128 weight rows (n) x BT tokens (m), one K-group (128) per MMA step.  The MMA runs
// "weight-stationary": the tensor core's A operand (M = 128) is the weight tile held in
// tensor memory, its B operand (N = BT) the token tile in shared memory, so a 16-token
// decode still uses the full 128-row MMA.
//
// Persistent CTAs, one per SM, walk a list of segments (tile, K-group range):
//   tile mode     whole tiles, round-robin over the CTAs (many tiles);
//   stream-K      the tiles' K-stages are cut into equal contiguous ranges, one per CTA, so
//                 every SM streams the same number of bytes (few tiles: decode, small M);
//                 with at least two CTAs per tile, every tile is split the same number of
//                 ways.  A tile covered by several CTAs is finished by the CTA holding its
//                 first stage, which adds the others' fp32 parts in CTA order
//                 (deterministic).  The parts travel through global memory (a release
//                 counter the owner polls) or, for 16- and 32-token tiles split 2-4 ways,
//                 inside a thread-block cluster: the partners write them into the owner's
//                 shared memory with st.async, counted in bytes on one of its mbarriers.
// Roles:
//   warp 0      TMA producer: packed W tile, one [128 x 128 B] box per two K-groups (a stage
//               holds two K-groups, four for tiles of at most 32 tokens), and
//               the token tile -- packed [BT x 128 B], or, in the expanded-activation mode,
//               one [BT x 128 B] int8 tile per group straight into the MMA operand slot.
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma kind::i8 (K = 32 each) per group
//               into a tensor-memory slot; one exact int32 partial per group.
//   warps 2..5  converters (one warpgroup): nibbles -> int8 in registers.  The weight row
//               of each thread goes to tensor memory (tcgen05.st); packed token rows go to
//               shared memory in the 128-byte-swizzled K-major operand layout.
//   then        epilogue (8 warps): tcgen05.ld of a group's partials while the next
//               groups' MMAs run, fp32 scale by sa*sw and accumulate in registers (packed
//               f32x2 math); fp16 output.  Each epilogue thread also fetches the scales it
//               needs, one block of 8 groups ahead (its weight row's sw; one token's sa,
//               shared with the other threads of its team through a small transposed
//               buffer).  Narrow tiles run two teams of 4 warps on alternate hand-off units.
// A warp reaches tensor-memory lanes 32*(warp % 4) .. +31 only, so each group of four
// consecutive warps covers the 128 lanes once.
//
// Nibble expansion: for a 32-bit word w of 8 packed nibbles, (w << 4) & 0xF0F0F0F0 holds
// 16*q for the 4 even k and w & 0xF0F0F0F0 16*q for the 4 odd k, as signed bytes.  Both
// operands get the same within-group K order (even k of a word, then odd k), so each
// group's sum is unchanged; the tensor core returns 256*P_g exactly (|256 P_g| <= 2^21),
// and the factor 1/256 is folded into the weight scale.  The expanded activations written
// by the quantizer use the same order and values (16*q).
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "ptx.cuh"
#include "quantize.cuh"

namespace apex {

enum GemmMode : int { MODE_PACKED = 0, MODE_AQ8 = 1, MODE_DUMP = 2 };

struct GemmArgs {
  int M, N, K;
  int gw;            // weight group (multiple of 128 dividing K)
  int gpg_shift;     // log2(gw / 128) when that is a power of two, else -1
  int G;             // K / 128
  int Gw;            // K / gw
  int tiles_n, tiles_m, T;   // tiles (n fastest)
  int S;             // K-stages per tile
  int kps;           // K-groups per stage (stage_groups(BT))
  int TS;            // T * S
  int P;             // persistent CTAs (gridDim.x)
  int streamk;       // 1: contiguous stage ranges per CTA; 0: whole tiles round-robin
  int cluster;       // >1: every tile is split over `cluster` consecutive CTAs launched as one
                     // thread-block cluster, which add their parts in the owner's shared
                     // memory (max_cluster(BT) at most); 1: parts go through global memory
  int sa_vec;        // sa rows readable as 16-byte vectors of 8 groups
  int sw_vec;        // sw rows readable as 16-byte vectors of 8 groups (gw == 128)
  const __half* sa;  // [M][G]
  const __half* sw;  // [N][Gw]
  __half* y;         // [M][N], or null when only the quantized output is wanted
  // Optional quantized output (null: none): Y's fp16 values quantized as the next layer's
  // activations, one scale per token per 128 outputs (N % 128 == 0).  qexp 0: packed
  // nibbles [M][N/2]; 1: the expanded operand form [M][N] (16*q bytes, GEMM K order).
  uint8_t* qout;
  __half* qscale;    // [M][N/128]
  int qexp;
  float* part;       // stream-K partial tiles [P][BT][128] fp32 (one per CTA)
  unsigned* counters;  // [T] arrival counters of split tiles (zero between calls)
  int32_t* dump;     // [G][M][N] per-group partials (debug kernel only)
  unsigned long long wait_ns;
  int withhold;      // test hook: the producer never loads this stage (-1: off)
  // Optional timeline trace (null: off), for the first trace_ctas CTAs:
  // SM clock stamps (clock64) [cta][role][step] with roles 0 producer issue, 1 converter
  // done and 4 converter inputs ready (per stage), 2 MMA issued, 3
  // epilogue done, 6 MMA inputs ready, 7 epilogue inputs ready, 8 MMA waits returned and
  // 9 MMAs issued before their commits (per K-group);
  // [cta][5][0..1] = %globaltimer at start / end, [cta][5][2] = the SM the CTA ran on,
  // [cta][5][3] = clock64 at start, [cta][5][4..5] = producer loop entry / first segment.
  unsigned long long* trace;
  int trace_ctas;
  int trace_steps;
};

constexpr int kTraceRoles = 16;

// clock64 into trace slot [cta][role][step] (used for the prologue marks of role 5).
__device__ __forceinline__ void trace_stamp_at(const GemmArgs& a, int role, int step) {
  if (a.trace == nullptr) return;
  const int cta = blockIdx.x;
  if (cta >= a.trace_ctas || step >= a.trace_steps) return;
  a.trace[((size_t)cta * kTraceRoles + role) * a.trace_steps + step] = clock_cycles();
}

__device__ __forceinline__ void trace_stamp(const GemmArgs& a, int role, int step) {
  if (a.trace == nullptr) return;
  const int cta = blockIdx.x;
  if (cta >= a.trace_ctas || step >= a.trace_steps) return;
  a.trace[((size_t)cta * kTraceRoles + role) * a.trace_steps + step] =
      role == 5 ? globaltimer_ns() : clock_cycles();
}

// K-groups per pipeline stage: narrow tiles move four groups per stage (two 128-byte TMA
// boxes of packed weights), so the per-stage hand-off costs are spread over more MMAs.
__host__ __device__ constexpr int stage_groups(int bt) { return bt <= 32 ? 4 : 2; }

// Largest cluster whose partial tiles (fp32 [BT][128] per partner) the owner CTA can take
// in shared memory: the narrow tiles of decode-sized batches.
__host__ __device__ constexpr int max_cluster(int bt) { return bt == 16 ? 4 : bt == 32 ? 2 : 1; }

template <int BT, int MODE, bool QOUT = false>
struct GemmCfg {
  static constexpr bool AQ8 = MODE == MODE_AQ8;
  static constexpr int BM = 128;
  static constexpr int KPS = stage_groups(BT);                     // K-groups per packed stage
  static constexpr int NBOX = KPS / 2;                             // 128-byte boxes per stage
  // operand slots (per group): expanded weight tile (tensor or shared memory) + token tile
  // (16-token tiles: three hand-off units, so the converters can fill one while the MMAs of
  // the two before it are still running; 12 x 32 + 8 x 16 columns fill the tensor memory)
  static constexpr int NX = BT >= 128 ? (AQ8 ? 6 : 4) : BT == 16 ? 12 : 8;
  static constexpr int NSLOT = BT >= 128 ? (AQ8 ? 2 : 3) : KPS == 4 ? 8 : 4;
  // Epilogue: 8 warps.  Wide tiles split the 128 columns in two halves; narrow tiles run
  // two teams of 4 warps that take alternate hand-off units (so one team's TMEM loads and
  // waits overlap the other's arithmetic) and add their sums at the end of a segment.
  static constexpr int EPI_WARPS = 8;
  static constexpr int TEAMS = BT >= 128 ? 1 : 2;
  static constexpr int CPT = BT >= 128 ? 64 : BT;  // columns per epilogue thread
  // converter warpgroups (a second one, with 18 warps, leaves 96 registers a thread and
  // spills in the epilogue: slower)
  static constexpr int CWG = 1;
  static constexpr int CONV0 = 2;                  // first converter warp
  static constexpr int EPI0 = CONV0 + 4 * CWG;     // first epilogue warp
  static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
  static constexpr int W_COL0 = 0;
  static constexpr int D_COL0 = NX * 32;
  static constexpr int TMEM_USED = D_COL0 + NSLOT * BT;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "tensor memory budget");
  static constexpr int PKW = BM * 64 * KPS;              // [BM rows][128 B], 128-byte swizzle
  static constexpr int PKA = AQ8 ? 0 : BT * 64 * KPS;   // [BT rows][128 B], 128-byte swizzle
  static constexpr int PK_STAGE = PKW + PKA;
  static constexpr int XA = BT * 128;                    // one group's int8 token tile
  // token scales: per team, 2 blocks x [8 groups][BT] fp32
  static constexpr int SAT = 2 * TEAMS * 8 * BT * 4;
  static constexpr int RED = TEAMS == 2 ? CPT * BM * 4 : 0;   // second team's sums [CPT][BM]
  // partners' partial tiles, received by a cluster's owner: [partner][BM rows][BT] fp32
  static constexpr int MAXCL = max_cluster(BT);
  static constexpr int RCV = (MAXCL - 1) * BT * BM * 4;
  static constexpr int FIXED = NX * XA + SAT + RED + RCV + 4096;
  static constexpr int NP_FIT = (200 * 1024 - FIXED) / PK_STAGE;
  static constexpr int NP = NP_FIT > 12 ? 12 : (NP_FIT < 2 ? 2 : NP_FIT);  // packed stages
  static constexpr int OFF_PK = 0;
  static constexpr int OFF_XA = OFF_PK + NP * PK_STAGE;
  static constexpr int OFF_SAT = OFF_XA + NX * XA;
  static constexpr int OFF_RED = OFF_SAT + SAT;
  static constexpr int OFF_RCV = OFF_RED + RED;
  // the quantized output's fp16 tile [BT tokens][BM rows] on its way from row-per-thread to
  // token-per-thread: narrow tiles stage it in the second team's sum buffer (idle by then),
  // wide tiles get a buffer of their own (left out of the stage budget above)
  static constexpr int STG = QOUT && TEAMS == 1 ? BT * BM * 2 : 0;
  static_assert(!QOUT || TEAMS == 1 || RED >= BT * BM * 2, "staging in the sum buffer");
  static constexpr int OFF_STG = OFF_RCV + RCV;
  static constexpr int OFF_BAR = OFF_STG + STG;
  // Hand-off unit: the groups that pass between converters, MMA and epilogue under one
  // barrier phase -- a whole stage for narrow tiles (the MMA issue loop is short on work
  // per group there), a single group for wide ones (whose partial slots fill TMEM).
  static constexpr int GPB = BT <= 64 ? KPS : 1;
  static constexpr int NXU = NX / GPB;      // operand hand-off units in flight
  static constexpr int NDU = NSLOT / GPB;   // partial hand-off units in flight
  static_assert(NX % GPB == 0 && NSLOT % GPB == 0, "slots come in whole units");
  static_assert(GPB == 1 || CWG * (KPS / CWG) == KPS, "converter split");
  static constexpr int NBAR = 2 * NP + 2 * NXU + NDU + 2;
  // one MMA-completion barrier per operand unit also tells the epilogue that the unit's
  // partials are ready, which needs every partial slot to be reused no sooner than its
  // operand slot
  static_assert(NDU <= NXU, "partial units cannot outnumber operand units");
  // operand slot of group j of stage q (flat group index gi)
  static __device__ __forceinline__ int slot(int q, int gi, int j) {
    return GPB == 1 ? gi % NX : (q % NXU) * GPB + j;
  }
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  static_assert(PK_STAGE % 1024 == 0 && XA % 1024 == 0, "stage alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t expand_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t expand_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// The 8 fp16 scales of groups gbeg .. gbeg+7 of one row, as raw bits (zeros outside
// [glo, ghi)).  vec: one 16-byte load (gbeg a multiple of 8, 16-byte aligned rows, weight
// group == 128).  Otherwise the scale of group g is base[row_off + g / gpg] (gpg = K-groups
// per scale group, gpg_shift = log2(gpg) when it is a power of two, else -1); when a scale
// group covers 8 groups or more, each distinct scale of the block is loaded once.
__device__ __forceinline__ uint4 load_scale_block(const __half* base, size_t row_off, int gbeg,
                                                  int glo, int ghi, bool vec, int gpg,
                                                  int gpg_shift) {
  if (vec) return __ldg(reinterpret_cast<const uint4*>(base + row_off + gbeg));
  const int lo = max(gbeg, glo), hi = min(gbeg + 8, ghi);   // groups of the block in use
  uint32_t h[8];
  if (gpg >= 8 || lo >= hi) {
    // at most two scale groups meet the block
    const int s0 = lo / gpg, s1 = (hi - 1) / gpg;
    const uint32_t v0 = lo < hi ? __half_as_ushort(base[row_off + s0]) : 0u;
    const uint32_t v1 = (lo < hi && s1 != s0) ? __half_as_ushort(base[row_off + s1]) : v0;
    const int split = (s0 + 1) * gpg;   // first group of the second scale group
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int g = gbeg + j;
      h[j] = (g >= lo && g < hi) ? (g < split ? v0 : v1) : 0u;
    }
  } else if (gpg_shift >= 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int g = gbeg + j;
      h[j] = (g >= lo && g < hi) ? __half_as_ushort(base[row_off + (g >> gpg_shift)]) : 0u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int g = gbeg + j;
      h[j] = (g >= lo && g < hi) ? __half_as_ushort(base[row_off + g / gpg]) : 0u;
    }
  }
  return make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                    h[6] | (h[7] << 16));
}

__device__ __forceinline__ float half_of(const uint4& v, int j) {
  const uint32_t w = j < 2 ? v.x : j < 4 ? v.y : j < 6 ? v.z : v.w;
  return __half2float(__ushort_as_half((uint16_t)((j & 1) ? (w >> 16) : (w & 0xFFFFu))));
}

// ------------------------------------------------------------------ work distribution

struct Seg {
  int t;    // tile
  int gb;   // first K-group
  int ge;   // one past the last K-group
};

// First stage-unit of CTA c under the stream-K partition (32-bit: the host only picks
// stream-K when P * T * S < 2^31).
__device__ __forceinline__ int sk_u0(const GemmArgs& a, int c) {
  return (int)((unsigned)c * (unsigned)a.TS / (unsigned)a.P);
}

// CTA owning stage-unit u under the stream-K partition.
__device__ __forceinline__ int sk_owner(const GemmArgs& a, int u) {
  return (int)((((unsigned)u + 1u) * (unsigned)a.P - 1u) / (unsigned)a.TS);
}

// k-th segment of this CTA; false when there is none.
__device__ __forceinline__ bool get_seg(const GemmArgs& a, int k, Seg& sg) {
  const int c = blockIdx.x;
  if (!a.streamk) {
    const int t = c + k * a.P;
    if (t >= a.T) return false;
    sg.t = t;
    sg.gb = 0;
    sg.ge = a.G;
    return true;
  }
  const int u0 = sk_u0(a, c), u1 = sk_u0(a, c + 1);
  if (u0 >= u1) return false;
  const int tf = u0 / a.S, tl = (u1 - 1) / a.S;
  const int t = tf + k;
  if (t > tl) return false;
  const int sb = t == tf ? u0 - tf * a.S : 0;
  const int se = t == tl ? (u1 - 1) - tl * a.S + 1 : a.S;
  sg.t = t;
  sg.gb = sb * a.kps;
  sg.ge = min(se * a.kps, a.G);
  return true;
}

// QOUT: the quantized output (args.qout) is written; a separate instantiation, so plain
// GEMMs carry none of its code.
template <int BT, int MODE, bool QOUT = false>
__global__ void __launch_bounds__(GemmCfg<BT, MODE, QOUT>::THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmA, const GemmArgs args) {
  using C = GemmCfg<BT, MODE, QOUT>;
  constexpr bool DUMP = MODE == MODE_DUMP;
  constexpr bool AQ8 = C::AQ8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* pk = smem + C::OFF_PK;
  uint8_t* xa = smem + C::OFF_XA;
  float* s_sat = reinterpret_cast<float*>(smem + C::OFF_SAT);
  float* s_red = reinterpret_cast<float*>(smem + C::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pk_full = bars;
  uint64_t* pk_empty = pk_full + C::NP;
  uint64_t* x_full = pk_empty + C::NP;
  // g_done[s]: the MMAs of the group in operand slot s have completed -- its operand slot
  // is free again and its partial is in tensor memory (one commit serves both waiters)
  uint64_t* g_done = x_full + C::NXU;
  uint64_t* d_empty = g_done + C::NXU;
  uint64_t* mma_done = d_empty + C::NDU;
  uint64_t* rcv_full = mma_done + 1;   // a cluster owner: every partner's part has landed
  float* s_rcv = reinterpret_cast<float*>(smem + C::OFF_RCV);
  uint8_t* s_stg = C::TEAMS == 2 ? reinterpret_cast<uint8_t*>(s_red) : smem + C::OFF_STG;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  int* s_abort = reinterpret_cast<int*>(smem + C::OFF_MISC + 4);
  int* s_last = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  int* s_never = reinterpret_cast<int*>(smem + C::OFF_MISC + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t lim = args.wait_ns;

  if (threadIdx.x == 0 && args.trace != nullptr && (int)blockIdx.x < args.trace_ctas &&
      args.trace_steps > 6)
    args.trace[((size_t)blockIdx.x * kTraceRoles + 5) * args.trace_steps + 6] = globaltimer_ns();
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NP; ++i) {
      mbar_init(smem_u32(&pk_full[i]), 1);
      mbar_init(smem_u32(&pk_empty[i]), C::CWG);   // one elected arrival per warpgroup
    }
    for (int i = 0; i < C::NXU; ++i) {
      mbar_init(smem_u32(&x_full[i]), C::CWG);     // one elected arrival per warpgroup
      mbar_init(smem_u32(&g_done[i]), 1);
    }
    for (int i = 0; i < C::NDU; ++i) {
      // one arrival per epilogue warp (one elected arrival per team for whole-stage units)
      mbar_init(smem_u32(&d_empty[i]), C::GPB == 1 ? C::EPI_WARPS : 1);
    }
    mbar_init(smem_u32(mma_done), 1);
    mbar_init(smem_u32(rcv_full), 1);
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
  // A split tile's CTAs may form one cluster, whose partners write into the owner's shared
  // memory at the end.  Announce here that this CTA's barriers are initialised; the
  // matching wait comes before the first remote access, long after, so it costs nothing.
  const bool clustered = C::MAXCL > 1 && !DUMP && args.cluster > 1;
  bool cl_waited = false;   // this thread has waited for that announcement
  if (clustered) cluster_arrive();
  // Launched as a programmatic dependent: the prologue above overlaps the previous grid's
  // tail.  The roles that touch global memory (producer, epilogue) wait for that grid
  // before their first access.
  grid_dep_launch();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(s_tmem);
  volatile int* abort_flag = s_abort;
  volatile int* never = s_never;
  if (threadIdx.x == 0) {
    trace_stamp(args, 5, 0);
    if (args.trace != nullptr && args.trace_steps > 3 && (int)blockIdx.x < args.trace_ctas) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      args.trace[((size_t)blockIdx.x * kTraceRoles + 5) * args.trace_steps + 2] = smid;
      args.trace[((size_t)blockIdx.x * kTraceRoles + 5) * args.trace_steps + 3] = clock_cycles();
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (converged); lane 0 issues.
    int q = 0, i = 0, last = -1;   // flat stage / group counters of this CTA
    bool ok = true;
    Seg sg;
    if (lane == 0) trace_stamp_at(args, 5, 4);
    grid_dep_wait();
    for (int k = 0; ok && get_seg(args, k, sg); ++k) {
      if (lane == 0 && k == 0) trace_stamp_at(args, 5, 5);
      const int n0 = (sg.t % args.tiles_n) * C::BM;
      const int m0 = (sg.t / args.tiles_n) * BT;
      for (int g = sg.gb; g < sg.ge; g += C::KPS, ++q) {
        const int nk = min(C::KPS, sg.ge - g);
        const int st = q % C::NP;
        const uint32_t pe_par = ((uint32_t)(q / C::NP) & 1u) ^ 1u;
        if constexpr (AQ8) {   // the token tiles land in the operand slots themselves
          const int u0 = C::GPB == 1 ? i : q;   // the stage's first hand-off unit
          ok = mbar_wait2(smem_u32(&pk_empty[st]), pe_par, smem_u32(&g_done[u0 % C::NXU]),
                          ((uint32_t)(u0 / C::NXU) & 1u) ^ 1u, lim, abort_flag);
          if constexpr (C::GPB == 1) {
            for (int j = 1; j < nk && ok; ++j)
              ok = mbar_wait(smem_u32(&g_done[(i + j) % C::NXU]),
                             ((uint32_t)((i + j) / C::NXU) & 1u) ^ 1u, lim, abort_flag);
          }
        } else {
          ok = mbar_wait(smem_u32(&pk_empty[st]), pe_par, lim, abort_flag);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (q == args.withhold) {
          i += nk;
          continue;
        }
        if (lane == 0) {
          const uint32_t fb = smem_u32(&pk_full[st]);
          const int nb = (nk + 1) >> 1;   // 128-byte boxes that hold the stage's groups
          mbar_arrive_expect_tx(fb, nb * (C::BM * 128) + (AQ8 ? nk * C::XA : nb * BT * 128));
          for (int b = 0; b < nb; ++b)
            tma_load_2d(smem_u32(pk + st * C::PK_STAGE + b * (C::BM * 128)), &tmW, fb,
                        (g + 2 * b) * 64, n0);
          if constexpr (AQ8) {
            for (int j = 0; j < nk; ++j)
              tma_load_2d(smem_u32(xa + C::slot(q, i + j, j) * C::XA), &tmA, fb, (g + j) * 128,
                          m0);
          } else {
            for (int b = 0; b < nb; ++b)
              tma_load_2d(smem_u32(pk + st * C::PK_STAGE + C::PKW + b * (BT * 128)), &tmA, fb,
                          (g + 2 * b) * 64, m0);
          }
          trace_stamp(args, 0, q);
        }
        __syncwarp();
        last = q;
        i += nk;
      }
    }
    // Never leave the CTA with bulk copies in flight: wait for the last stages issued.
    for (int s = (last - C::NP + 1 > 0 ? last - C::NP + 1 : 0); s <= last; ++s) {
      if (s == args.withhold) continue;
      mbar_wait(smem_u32(&pk_full[s % C::NP]), (uint32_t)(s / C::NP) & 1u, lim, never);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (converged); lane 0 issues the MMAs and commits.
    constexpr uint32_t idesc = idesc_i8(128, BT);
    int i = 0, q = 0;   // flat group / stage counters of this CTA
    bool ok = true;
    Seg sg;
    for (int k = 0; ok && get_seg(args, k, sg); ++k) {
      for (int g = sg.gb; ok && g < sg.ge; g += C::KPS, ++q) {
        const int nk = min(C::KPS, sg.ge - g);
        // the stage's hand-off units: one per group, or the whole stage
        for (int j0 = 0; j0 < nk; j0 += C::GPB) {
          const int u = C::GPB == 1 ? i + j0 : q;
          const int nu = min(C::GPB, nk - j0);
          const int xu = u % C::NXU, du = u % C::NDU;
          ok = mbar_wait2(smem_u32(&x_full[xu]), (uint32_t)(u / C::NXU) & 1u,
                          smem_u32(&d_empty[du]), ((uint32_t)(u / C::NDU) & 1u) ^ 1u, lim,
                          abort_flag);
          if (lane == 0) trace_stamp(args, 8, i + j0);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            trace_stamp(args, 6, i + j0);
            for (int t = 0; t < nu; ++t) {
              const int xs = xu * C::GPB + t;
              const uint32_t d = tbase + C::D_COL0 + (du * C::GPB + t) * BT;
              const uint64_t b0 = smem_desc_k_sw128(smem_u32(xa + xs * C::XA));
              const uint32_t a0 = tbase + C::W_COL0 + xs * 32;
#pragma unroll
              for (int j = 0; j < 4; ++j)
                umma_i8_ts(d, a0 + j * 8, b0 + (uint64_t)(j * 2), idesc, j > 0 ? 1u : 0u);
            }
            trace_stamp(args, 9, i + j0);
            umma_commit(smem_u32(&g_done[xu]));
            trace_stamp(args, 2, i + j0);
          }
          __syncwarp();
        }
        i += nk;
      }
    }
    if (lane == 0) umma_commit(smem_u32(mma_done));
    __syncwarp();
    mbar_wait(smem_u32(mma_done), 0u, lim, never);
    __syncwarp();
  } else if (warp >= C::CONV0 && warp < C::CONV0 + 4 * C::CWG) {
    // ------------------------------------------------------------ converters
    // Warpgroup w expands the K-groups j of every stage with j % CWG == w, so with two
    // warpgroups both work on each stage at once, one group each.
    const int cwg = (warp - C::CONV0) >> 2;
    const uint32_t CB = cwg == 0 ? 2 : 6;              // this warpgroup's named barrier
    const int row = 32 * (warp & 3) + lane;            // this thread's W row (TMEM lane)
    const int ct = threadIdx.x - 32 * (C::CONV0 + 4 * cwg);  // 0..127, for the token rows
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    constexpr int JPW = C::KPS / C::CWG;                   // groups per warpgroup per stage
    constexpr int NITG = AQ8 ? 0 : BT * 8 / 128;           // token 8-byte units per thread
    int q = 0, i = 0;
    bool ok = true;
    Seg sg;
    for (int k = 0; ok && get_seg(args, k, sg); ++k) {
      for (int g = sg.gb; g < sg.ge; g += C::KPS, ++q) {
        const int st = q % C::NP;
        const int nk = min(C::KPS, sg.ge - g);
        // The stage's bytes, and the operand slots it fills (their previous use done).  One
        // warp waits; the others park in the hardware barrier below, where barrier events
        // do not wake them.
        const uint32_t pf_par = (uint32_t)(q / C::NP) & 1u;
        if (ct < 32) {
          if constexpr (C::GPB != 1) {
            ok = mbar_wait2(smem_u32(&pk_full[st]), pf_par, smem_u32(&g_done[q % C::NXU]),
                            ((uint32_t)(q / C::NXU) & 1u) ^ 1u, lim, abort_flag);
          } else {
            ok = mbar_wait2(smem_u32(&pk_full[st]), pf_par, smem_u32(&g_done[i % C::NXU]),
                            ((uint32_t)(i / C::NXU) & 1u) ^ 1u, lim, abort_flag);
            for (int j = 1; j < nk; ++j)
              ok = ok && mbar_wait(smem_u32(&g_done[(i + j) % C::NXU]),
                                   ((uint32_t)((i + j) / C::NXU) & 1u) ^ 1u, lim, abort_flag);
          }
        }
        // one decision for the whole warpgroup, so none of it can be left at the barrier
        // below when another part gives up
        ok = !bar_red_or(CB, 128, !ok);
        tc_fence_after();   // tensor-memory writes below come after the slots' last reads
        if (!ok) break;
        if (lane == 0 && (warp & 3) == 2) trace_stamp(args, 4, q);
        const uint8_t* pw = pk + st * C::PK_STAGE;
        // All shared-memory reads first, so their latencies overlap.  Packed W: group j of
        // the stage lies in 128-byte box j / 2, chunks 4 (j % 2) .. +3 of the row, with the
        // 16-byte chunk c of a box row stored at c ^ (row & 7).
        uint4 wraw[4 * JPW];
        uint2 araw[JPW * NITG + 1];
#pragma unroll
        for (int jj = 0; jj < JPW; ++jj) {
          const int j = cwg + C::CWG * jj;
          if (j < nk) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              wraw[4 * jj + c] = *reinterpret_cast<const uint4*>(
                  pw + (j >> 1) * (C::BM * 128) + row * 128 +
                  (((4 * (j & 1) + c) ^ (row & 7)) << 4));
            if constexpr (!AQ8) {
              const uint8_t* pa = pw + C::PKW;
#pragma unroll
              for (int x = 0; x < NITG; ++x) {
                // unit (v, u): token row v, 8-byte unit u of its 64 packed bytes.  Rows r
                // and r+4 of an 8-row block share a load phase, so their 16-byte chunks
                // fall in different banks.
                const int it = ct + 128 * x;
                const int v = it >> 3, u = it & 7;
                const int r = (v & ~7) | ((v & 1) << 2) | ((v >> 1) & 3);
                araw[jj * NITG + x] = *reinterpret_cast<const uint2*>(
                    pa + (j >> 1) * (BT * 128) + r * 128 +
                    (((4 * (j & 1) + (u >> 1)) ^ (r & 7)) << 4) + ((u & 1) << 3));
              }
            }
          }
        }
#pragma unroll
        for (int jj = 0; jj < JPW; ++jj) {
          const int j = cwg + C::CWG * jj;
          if (j >= nk) continue;
          const int xs = C::slot(q, i + j, j);
          {
            uint32_t e0[16], e1[16];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 a = wraw[4 * jj + c], b = wraw[4 * jj + 2 + c];
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
          if constexpr (!AQ8) {
#pragma unroll
            for (int x = 0; x < NITG; ++x) {
              const int it = ct + 128 * x;
              const int v = it >> 3, u = it & 7;
              const int r = (v & ~7) | ((v & 1) << 2) | ((v >> 1) & 3);
              const uint2 w2 = araw[jj * NITG + x];
              *reinterpret_cast<uint4*>(xa + xs * C::XA + r * 128 + ((u ^ (r & 7)) << 4)) =
                  make_uint4(expand_lo(w2.x), expand_hi(w2.x), expand_lo(w2.y),
                             expand_hi(w2.y));
            }
          }
        }
        if constexpr (!AQ8) fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        // every converter thread's writes are ordered before one elected arrival (fewer
        // barrier events: each one wakes every suspended waiter of the CTA)
        named_bar_sync(CB, 128);
        if (ct == 0) {
          mbar_arrive(smem_u32(&pk_empty[st]));
          if constexpr (C::GPB != 1) {
            mbar_arrive(smem_u32(&x_full[q % C::NXU]));
          } else {
#pragma unroll
            for (int jj = 0; jj < JPW; ++jj) {
              const int j = cwg + C::CWG * jj;
              if (j < nk) mbar_arrive(smem_u32(&x_full[(i + j) % C::NXU]));
            }
          }
        }
        if (lane == 0 && (warp & 3) == 2) trace_stamp(args, 1, q);
        if (lane == 0) trace_stamp(args, 11 + (warp & 3), q);
        i += nk;
      }
    }
  } else if (warp >= C::EPI0) {
    // ------------------------------------------------------------ epilogue
    grid_dep_wait();   // scales, outputs and split-K scratch are global memory
    const int et = threadIdx.x - 32 * C::EPI0;
    const int ew = (warp - C::EPI0) >> 2;
    const int h = C::TEAMS == 1 ? ew : 0;          // column block (64 columns) of this warp
    const int team = C::TEAMS == 2 ? ew : 0;       // hand-off units u with u % 2 == team
    const int row = 32 * (warp & 3) + lane;        // TMEM lane = weight row in the tile
    const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
    constexpr int NE = C::EPI_WARPS * 32;
    // the tile flush: the whole epilogue, or the first team alone (barrier 5)
    constexpr int NF = C::TEAMS == 2 ? 128 : NE;
    constexpr uint32_t FB = C::TEAMS == 2 ? 5 : 1;
    const uint32_t TB = 3 + team;                  // this team's unit barrier
    // token of this thread for the token-scale staging (each team stages its own copy)
    const int tt = C::TEAMS == 2 ? (et & 127) : et;
    const int M = args.M, N = args.N;
    const bool sa_vec = args.sa_vec != 0, sw_vec = args.sw_vec != 0;
    // cluster mode: every tile is split over exactly `cluster` CTAs, the owner at rank 0
    bool expected = false;   // an owner: the parts' byte count is armed on rcv_full
    bool received = false;   // an owner: its partners' parts are in its shared memory
    // Pairs (2-CTA clusters, plain output): each CTA finishes half of the tile's tokens
    const bool PAIRS = !QOUT && args.cluster == 2;
    constexpr int HALF = C::CPT / 2;
    bool sent = false;       // a pair: this CTA's other half went to its peer

    // Scales of the 8-group block starting at gb8 of segment sg (this thread's token / row).
    auto block_scales = [&](const Seg& sg, int gb8, uint4& sa, uint4& sw) {
      sa = make_uint4(0, 0, 0, 0);
      sw = make_uint4(0, 0, 0, 0);
      if (DUMP) return;
      const int mt = (sg.t / args.tiles_n) * BT + tt;
      const int nn = (sg.t % args.tiles_n) * C::BM + row;
      if (tt < BT && mt < M)
        sa = load_scale_block(args.sa, (size_t)mt * args.G, gb8, sg.gb, sg.ge, sa_vec, 1, 0);
      if (nn < N)
        sw = load_scale_block(args.sw, (size_t)nn * args.Gw, gb8, sg.gb, sg.ge, sw_vec,
                              args.gw / 128, args.gpg_shift);
    };

    float2 acc[C::CPT / 2];
    // the pair's exchange with compile-time column offsets (acc stays in registers): send the
    // columns [O, O + HALF) of acc to the peer, or add the received half into [O, O + HALF)
    auto pair_send = [&](auto o_c, uint32_t dst, uint32_t bar) {
      constexpr int O = decltype(o_c)::value;
#pragma unroll
      for (int e = 0; e < HALF; e += 4)
        st_async_v4(dst + 4u * e, acc[(O + e) / 2].x, acc[(O + e) / 2].y,
                    acc[(O + e) / 2 + 1].x, acc[(O + e) / 2 + 1].y, bar);
    };
    auto pair_add_write = [&](auto o_c, int m0t, int nn, bool nvalid_) {
      constexpr int O = decltype(o_c)::value;
      const float4* src = reinterpret_cast<const float4*>(s_rcv + (size_t)row * HALF);
#pragma unroll
      for (int e = 0; e < HALF; e += 4) {
        const float4 v = src[e / 4];
        acc[(O + e) / 2].x += v.x;
        acc[(O + e) / 2].y += v.y;
        acc[(O + e) / 2 + 1].x += v.z;
        acc[(O + e) / 2 + 1].y += v.w;
      }
#pragma unroll
      for (int e = 0; e < HALF; ++e) {
        const int m = m0t + h * C::CPT + O + e;
        const float v = ((O + e) & 1) ? acc[(O + e) / 2].y : acc[(O + e) / 2].x;
        if (m < M && nvalid_) args.y[(size_t)m * N + nn] = __float2half_rn(v);
      }
    };
    // Where the finished tile is written: from one call site after the hand-off (always with
    // the quantized output; for 128-token tiles also without it, measured 2-3 % faster), or
    // in place at each hand-off path (narrow tiles: measured faster)
    constexpr bool ONE_WRITE = QOUT || BT >= 128;

    // The finished tile goes out as fp16 Y (when args.y is set) and, when args.qout is set,
    // as the next layer's quantized activations: for each token, the tile's 128 rows are
    // exactly one 128-wide K-group of that token's input to the next layer, so the group's
    // scale and codes are made here, from the fp16 values Y holds and with the rule of the
    // activation quantizer.  Every flushing thread calls it (NF threads, barrier FB).
    auto write_tile = [&](int m0t, int n0t) {
      const int n = n0t + row;
      if (args.y != nullptr) {
#pragma unroll
        for (int e = 0; e < C::CPT; ++e) {
          const int m = m0t + h * C::CPT + e;
          const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
          if (m < M && n < N) args.y[(size_t)m * N + n] = __float2half_rn(v);
        }
      }
      if constexpr (!QOUT) return;
      // The quantized output is made token by token.  The tile goes through shared memory
      // as fp16 [token][128 rows]; then TPT neighbouring threads take one token's 128
      // values, RPT each, find the group's absmax with a few shuffles and quantize with the
      // activation quantizer's own routines: one scale per token, independent divisions,
      // whole words stored.  The 16-byte chunks of a token's line are permuted (chunk c
      // lives at c ^ ((token * TPT + c / R8) & 7)) so that the row-per-thread writes and the
      // token-per-thread 16-byte reads both meet every bank once per phase.
      constexpr int TPT = NF / BT;               // threads per token
      constexpr int RPT = C::BM / TPT;           // values (the next layer's k) per thread
      constexpr int R8 = RPT / 8;                // their 16-byte chunks
      static_assert(NF % BT == 0 && 32 % TPT == 0 && R8 >= 2, "token-per-thread mapping");
      auto chunk_at = [&](int tok, int c) {
        return tok * (C::BM * 2) + ((c ^ ((tok * TPT + c / R8) & 7)) << 4);
      };
      // narrow tiles stage in the sum buffer: every thread has read its sums out of it
      if constexpr (C::TEAMS == 2) named_bar_sync(FB, NF);
#pragma unroll
      for (int e = 0; e < C::CPT; ++e) {
        const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
        *reinterpret_cast<__half*>(s_stg + chunk_at(h * C::CPT + e, row >> 3) +
                                   2 * (row & 7)) = __float2half_rn(v);
      }
      named_bar_sync(FB, NF);
      {
        const int tok = et / TPT, part = et % TPT;
        uint4 v[R8];
#pragma unroll
        for (int j = 0; j < R8; ++j)
          v[j] = *reinterpret_cast<const uint4*>(s_stg + chunk_at(tok, part * R8 + j));
        __half2 mx = __float2half2_rn(0.0f);
#pragma unroll
        for (int j = 0; j < R8; ++j) {
          const __half2* hv = reinterpret_cast<const __half2*>(&v[j]);
#pragma unroll
          for (int i = 0; i < 4; ++i) mx = __hmax2(mx, __habs2(hv[i]));
        }
        float am = fmaxf(__low2float(mx), __high2float(mx));
#pragma unroll
        for (int o = 1; o < TPT; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        const __half sc = group_scale(am);
        const QScale qs = make_qscale(__half2float(sc));
        const int m = m0t + tok;
        if (m < M) {
          if (args.qexp) {
            uint8_t* dst = args.qout + (size_t)m * N + n0t + part * RPT;
#pragma unroll
            for (int j = 0; j < R8; j += 2) {
              const uint2 x0 = quant_expand8(v[j], qs), x1 = quant_expand8(v[j + 1], qs);
              *reinterpret_cast<uint4*>(dst + 8 * j) = make_uint4(x0.x, x0.y, x1.x, x1.y);
            }
          } else {
            uint8_t* dst = args.qout + (size_t)m * (N / 2) + n0t / 2 + part * (RPT / 2);
            if constexpr (R8 == 2) {
              *reinterpret_cast<uint2*>(dst) =
                  make_uint2(quant_pack8(v[0], qs), quant_pack8(v[1], qs));
            } else {
#pragma unroll
              for (int j = 0; j < R8; j += 4)
                *reinterpret_cast<uint4*>(dst + 4 * j) =
                    make_uint4(quant_pack8(v[j], qs), quant_pack8(v[j + 1], qs),
                               quant_pack8(v[j + 2], qs), quant_pack8(v[j + 3], qs));
            }
          }
          if (part == 0) args.qscale[(size_t)m * (N / 128) + n0t / 128] = sc;
        }
      }
      named_bar_sync(FB, NF);   // the staging buffer is free again
    };
    // Narrow tiles pipeline the partial loads within a hand-off unit.
    constexpr bool PIPE = C::CPT == 16 && C::GPB > 1;
    bool ok = true, aborted = false;
    int i = 0;     // flat group counter of this CTA
    int u = 0;     // flat hand-off unit counter of this CTA
    int buf = 0;   // token-scale buffer in use
    Seg sg, nx;
    bool have = get_seg(args, 0, sg);
    uint4 sa_c = make_uint4(0, 0, 0, 0), sw_c = make_uint4(0, 0, 0, 0);
    if (have) block_scales(sg, sg.gb & ~7, sa_c, sw_c);
    for (int k = 0; have && !aborted; ++k) {
      const int n0 = (sg.t % args.tiles_n) * C::BM;
      const int m0 = (sg.t / args.tiles_n) * BT;
      const int n = n0 + row;
      const bool nvalid = n < N;
      // One weight group spans the whole segment: sw factors out of the sum.
      const bool hoist = (sg.gb * 128) / args.gw == ((sg.ge - 1) * 128) / args.gw;
      const bool have_next = get_seg(args, k + 1, nx);
#pragma unroll
      for (int e = 0; e < C::CPT / 2; ++e) acc[e] = make_float2(0.0f, 0.0f);
      float sw_hoisted = 0.0f;
      uint32_t pc[16];   // partials of the group in hand (units never straddle segments)
      for (int gb8 = sg.gb & ~7; gb8 < sg.ge; gb8 += 8) {
        // the next block's scales are in flight while this block is processed
        uint4 sa_n, sw_n;
        if (gb8 + 8 < sg.ge)
          block_scales(sg, gb8 + 8, sa_n, sw_n);
        else if (have_next)
          block_scales(nx, nx.gb & ~7, sa_n, sw_n);
        else
          sa_n = sw_n = make_uint4(0, 0, 0, 0);
        float* sat = s_sat + (buf * C::TEAMS + team) * 8 * BT;
        if (tt < BT) {
#pragma unroll
          for (int j = 0; j < 8; ++j) sat[j * BT + tt] = half_of(sa_c, j);
        }
        // token scales visible, one abort decision: per team, so that the two teams do not
        // wait for each other at every block (the segment end below joins them)
        aborted = C::TEAMS == 2 ? bar_red_or(TB, 128, !ok) : bar_red_or(1, NE, !ok);
        if (aborted) break;
        if (gb8 <= sg.gb) sw_hoisted = half_of(sw_c, sg.gb - gb8) * (1.0f / 256.0f);
        const int jb = max(sg.gb - gb8, 0), je = min(sg.ge - gb8, 8);
#pragma unroll 1
        for (int j = jb; j < je; ++j, ++i) {
          const int r = (gb8 + j - sg.gb) % C::GPB;   // position in its hand-off unit
          const bool unit_last = r == C::GPB - 1 || gb8 + j == sg.ge - 1;
          const int sl = (u % C::NDU) * C::GPB + r;
          if (C::TEAMS == 2 && (u & 1) != team) {   // the other team's unit
            if (unit_last) ++u;
            continue;
          }
          if (r == 0) {
            if constexpr (C::GPB == 1) {
              ok = mbar_wait(smem_u32(&g_done[u % C::NXU]), (uint32_t)(u / C::NXU) & 1u, lim,
                             abort_flag);
              ok = __all_sync(0xffffffffu, ok);
            } else {
              // one warp of the team waits; the others park in the team's hardware barrier
              if ((et & 127) < 32)
                ok = mbar_wait(smem_u32(&g_done[u % C::NXU]), (uint32_t)(u / C::NXU) & 1u,
                               lim, abort_flag);
              ok = !bar_red_or(TB, 128, !ok);   // one decision for the team
            }
            if (!ok) break;
            if (et == 0) trace_stamp(args, 7, i);
            tc_fence_after();
          }
          const float4* sab = reinterpret_cast<const float4*>(sat + j * BT + h * 64);
          const float swj = half_of(sw_c, j) * (1.0f / 256.0f);
          const float2 sw2 = make_float2(swj, swj);
          const uint32_t td = tbase + t_lane + C::D_COL0 + sl * BT + h * 64;
          // dequantise and accumulate 16 partials (columns cc*16 ..) of this group
          auto consume = [&](const uint32_t* p, int cc) {
            if constexpr (DUMP) {
              const int g = gb8 + j;
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int m = m0 + h * 64 + cc * 16 + e;
                if (m < M && nvalid)
                  args.dump[((size_t)g * M + m) * N + n] = static_cast<int32_t>(p[e]) >> 8;
              }
            } else {
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) {
                const float4 s4 = sab[cc * 4 + qq];
                const float2 pa =
                    make_float2((float)(int32_t)p[4 * qq + 0], (float)(int32_t)p[4 * qq + 1]);
                const float2 pb =
                    make_float2((float)(int32_t)p[4 * qq + 2], (float)(int32_t)p[4 * qq + 3]);
                float2 sa_a = make_float2(s4.x, s4.y), sa_b = make_float2(s4.z, s4.w);
                if (!hoist) {
                  sa_a = __fmul2_rn(sa_a, sw2);
                  sa_b = __fmul2_rn(sa_b, sw2);
                }
                acc[cc * 8 + 2 * qq] = __ffma2_rn(pa, sa_a, acc[cc * 8 + 2 * qq]);
                acc[cc * 8 + 2 * qq + 1] = __ffma2_rn(pb, sa_b, acc[cc * 8 + 2 * qq + 1]);
              }
            }
          };
          if constexpr (PIPE) {
            // the unit's first group is loaded here; every later one was loaded while the
            // group before it was being processed
            if (r == 0) {
              tmem_ld16_nowait(td, pc);
              tmem_ld_wait16(pc);
            }
            uint32_t pn[16];
            if (!unit_last) tmem_ld16_nowait(td + BT, pn);
            consume(pc, 0);
            if (!unit_last) {
              tmem_ld_wait16(pn);
#pragma unroll
              for (int e = 0; e < 16; ++e) pc[e] = pn[e];
            }
          } else {
#pragma unroll
            for (int cc = 0; cc < C::CPT / 16; ++cc) {
              uint32_t p[16];
              tmem_ld16(td + cc * 16, p);
              consume(p, cc);
            }
          }
          if (unit_last) {
            tc_fence_before();
            if constexpr (C::GPB == 1) {
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_u32(&d_empty[u % C::NDU]));
            } else {
              named_bar_sync(TB, 128);   // the team is done with the unit: one arrival
              if ((et & 127) == 0) mbar_arrive(smem_u32(&d_empty[u % C::NDU]));
            }
            ++u;
          }
          if (et == 0) trace_stamp(args, 3, i);
        }
        buf ^= 1;
        sa_c = sa_n;
        sw_c = sw_n;
      }
      // ---- segment finished: write the tile, or hand its partial to the fixup
      if (et == 0) trace_stamp(args, 15, 4 * k);
      aborted = bar_red_or(1, NE, aborted || !ok);   // every thread takes part, always
      if (aborted) break;
      if constexpr (C::TEAMS == 2 && !DUMP) {
        // the second team hands its sums to the first, which adds them (fixed order)
        if (team == 1) {
#pragma unroll
          for (int e = 0; e < C::CPT; ++e)
            s_red[e * C::BM + row] = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
        }
        bar_red_or(1, NE, false);
        if (team == 0) {
#pragma unroll
          for (int e = 0; e < C::CPT; e += 2) {
            acc[e / 2].x += s_red[e * C::BM + row];
            acc[e / 2].y += s_red[(e + 1) * C::BM + row];
          }
        }
      }
      if (!DUMP && team == 0) {
        if (hoist) {
          const float2 sh = make_float2(sw_hoisted, sw_hoisted);
#pragma unroll
          for (int e = 0; e < C::CPT / 2; ++e) acc[e] = __fmul2_rn(acc[e], sh);
        }
        const int cf = args.streamk ? sk_owner(args, sg.t * args.S) : (int)blockIdx.x;
        const int cl = args.streamk ? sk_owner(args, sg.t * args.S + args.S - 1) : (int)blockIdx.x;
        bool owner_done = false;   // this CTA holds the whole tile now: write it
        if (clustered && PAIRS) {
          // A pair finishes the tile half each: this CTA sends its sums of the other half's
          // tokens to its peer, adds the peer's sums of its own half and writes that half.
          // (Two addends: the result does not depend on which CTA adds.)
          const int cl_rank = (int)(blockIdx.x & 1u);
          if (et == 0)
            mbar_arrive_expect_tx(smem_u32(rcv_full), (uint32_t)(HALF * C::BM * 4));
          expected = true;
          cluster_wait();   // the peer's barriers are initialised
          cl_waited = true;
          {
            const uint32_t dst =
                cluster_map(smem_u32(s_rcv + (size_t)row * HALF), (uint32_t)(cl_rank ^ 1));
            const uint32_t bar = cluster_map(smem_u32(rcv_full), (uint32_t)(cl_rank ^ 1));
            if (cl_rank == 0) pair_send(std::integral_constant<int, HALF>{}, dst, bar);
            else pair_send(std::integral_constant<int, 0>{}, dst, bar);
          }
          sent = true;
          ok = mbar_wait_cluster(smem_u32(rcv_full), 0u, lim, abort_flag);
          received = ok;
          if (et == 0) trace_stamp(args, 15, 4 * k + 2);
          aborted = bar_red_or(FB, NF, !ok);
          if (aborted) break;
          if (cl_rank == 0) pair_add_write(std::integral_constant<int, 0>{}, m0, n, nvalid);
          else pair_add_write(std::integral_constant<int, HALF>{}, m0, n, nvalid);
        } else if (clustered) {
          // The parts meet in the owner's shared memory.  A partner sends its part after the
          // segment loop (below), on every path; the owner takes them here, adds them in
          // CTA order and writes the tile.
          if (blockIdx.x % (unsigned)args.cluster == 0) {
            if (et == 0)
              mbar_arrive_expect_tx(smem_u32(rcv_full),
                                    (uint32_t)((args.cluster - 1) * BT * C::BM * 4));
            expected = true;
            ok = mbar_wait_cluster(smem_u32(rcv_full), 0u, lim, abort_flag);
            received = ok;
            if (et == 0) trace_stamp(args, 15, 4 * k + 2);
            aborted = bar_red_or(FB, NF, !ok);
            if (aborted) break;
            for (int c = 1; c < args.cluster; ++c) {
              const float4* src = reinterpret_cast<const float4*>(
                  s_rcv + ((size_t)(c - 1) * C::BM + row) * C::CPT);
#pragma unroll
              for (int e = 0; e < C::CPT; e += 4) {
                const float4 v = src[e / 4];
                acc[e / 2].x += v.x;
                acc[e / 2].y += v.y;
                acc[e / 2 + 1].x += v.z;
                acc[e / 2 + 1].y += v.w;
              }
            }
            if constexpr (ONE_WRITE) {
              owner_done = true;
            } else {
#pragma unroll
              for (int e = 0; e < C::CPT; ++e) {
                const int m = m0 + h * C::CPT + e;
                const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
                if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(v);
              }
            }
          }
        } else if (cf == cl) {
          if constexpr (ONE_WRITE) {
            owner_done = true;
          } else {
#pragma unroll
            for (int e = 0; e < C::CPT; ++e) {
              const int m = m0 + h * C::CPT + e;
              const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
              if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(v);
            }
          }
        } else {
          // A split tile is finished by its owner, the CTA holding the tile's first stage:
          // that is always the owner's last segment, so the others (the CTAs after it, for
          // which the tile is their first segment) have published their parts by then or
          // are about to.  A non-owner stores its fp32 part in its one slot and counts
          // itself in; the owner waits for the count, then adds the parts in CTA order.
          if ((int)blockIdx.x != cf) {
            float* mine = args.part + (size_t)blockIdx.x * (BT * C::BM);
#pragma unroll
            for (int e = 0; e < C::CPT; ++e) {
              const int ml = h * 64 + e;
              mine[(size_t)ml * C::BM + row] = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
            }
            // the barrier collects every thread's stores; one thread releases them with
            // the count
            bar_red_or(FB, NF, false);
            if (et == 0) trace_stamp(args, 15, 4 * k + 1);
            if (et == 0) {
              fence_acq_rel_gpu();
              atomicAdd(&args.counters[sg.t], 1u);
            }
          } else {
            if (et == 0) {
              const unsigned need = (unsigned)(cl - cf);
              ok = counter_wait(&args.counters[sg.t], need, lim, abort_flag);
              trace_stamp(args, 15, 4 * k + 2);
            }
            aborted = bar_red_or(FB, NF, !ok);   // the other parts are visible to every thread
            if (aborted) break;
            // the other parts, added to this CTA's own in CTA order, NCH CTAs in flight
            constexpr int NCH = C::CPT >= 64 ? 1 : C::CPT >= 32 ? 2 : 4;
            for (int c = cf + 1; c <= cl; c += NCH) {
#pragma unroll
              for (int e0 = 0; e0 < C::CPT; e0 += 16) {
                float v[NCH][16];
#pragma unroll
                for (int cc = 0; cc < NCH; ++cc) {
                  const float* src = args.part + (size_t)min(c + cc, cl) * (BT * C::BM);
#pragma unroll
                  for (int e = 0; e < 16; ++e)
                    v[cc][e] = c + cc <= cl
                                   ? __ldcg(src + (size_t)(h * 64 + e0 + e) * C::BM + row)
                                   : 0.0f;
                }
#pragma unroll
                for (int cc = 0; cc < NCH; ++cc)
#pragma unroll
                  for (int e = 0; e < 16; e += 2) {
                    acc[(e0 + e) / 2].x += v[cc][e];
                    acc[(e0 + e) / 2].y += v[cc][e + 1];
                  }
              }
            }
            if constexpr (ONE_WRITE) {
              owner_done = true;
            } else {
#pragma unroll
              for (int e = 0; e < C::CPT; ++e) {
                const int m = m0 + h * C::CPT + e;
                const float v = (e & 1) ? acc[e / 2].y : acc[e / 2].x;
                if (m < M && nvalid) args.y[(size_t)m * N + n] = __float2half_rn(v);
              }
            }
            if (et == 0) args.counters[sg.t] = 0u;   // nobody else touches it in this launch
          }
        }
        if constexpr (ONE_WRITE) {
          if (owner_done) write_tile(m0, n0);   // the whole team takes it together
        }
      }
      if (et == 0) trace_stamp(args, 15, 4 * k + 3);
      have = have_next;
      sg = nx;
    }
    if (clustered && PAIRS && team == 0) {
      // a CTA that gave up before its segment's end still sends its half (whatever it holds),
      // so its peer's wait ends, and still takes its peer's half, so that no store into this
      // CTA's shared memory is in flight when it exits
      const int cl_rank = (int)(blockIdx.x & 1u);
      if (!sent) {
        if (!cl_waited) cluster_wait();
        cl_waited = true;
        const uint32_t dst =
            cluster_map(smem_u32(s_rcv + (size_t)row * HALF), (uint32_t)(cl_rank ^ 1));
        const uint32_t bar = cluster_map(smem_u32(rcv_full), (uint32_t)(cl_rank ^ 1));
        if (cl_rank == 0) pair_send(std::integral_constant<int, HALF>{}, dst, bar);
        else pair_send(std::integral_constant<int, 0>{}, dst, bar);
      }
      if (!received) {
        if (et == 0 && !expected)
          mbar_arrive_expect_tx(smem_u32(rcv_full), (uint32_t)(HALF * C::BM * 4));
        mbar_wait_cluster(smem_u32(rcv_full), 0u, 2 * lim, never);
      }
    } else if (clustered && team == 0) {
      const int cl_rank = (int)(blockIdx.x % (unsigned)args.cluster);
      if (cl_rank != 0) {
        // A partner's part (its one segment's sums; whatever it holds if the CTA gave up)
        // goes to the owner on every path, so the owner's wait below always ends.
        cluster_wait();   // the owner's barriers are initialised
        cl_waited = true;
        const uint32_t dst = cluster_map(
            smem_u32(s_rcv + ((size_t)(cl_rank - 1) * C::BM + row) * C::CPT), 0u);
        const uint32_t bar = cluster_map(smem_u32(rcv_full), 0u);
#pragma unroll
        for (int e = 0; e < C::CPT; e += 4)
          st_async_v4(dst + 4u * e, acc[e / 2].x, acc[e / 2].y, acc[e / 2 + 1].x,
                      acc[e / 2 + 1].y, bar);
        if (et == 0) trace_stamp(args, 15, 1);
      } else if (!received) {
        // an owner that gave up before its flush still takes its partners' parts, so that no
        // store into this CTA's shared memory is in flight when it exits
        if (et == 0 && !expected)
          mbar_arrive_expect_tx(smem_u32(rcv_full),
                                (uint32_t)((args.cluster - 1) * BT * C::BM * 4));
        mbar_wait_cluster(smem_u32(rcv_full), 0u, 2 * lim, never);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (clustered) {
    // No CTA of the cluster exits before its partners have issued their stores into its
    // shared memory.  Their arrival is counted on the owner's mbarrier, which the owner
    // waits for on every path, so this barrier orders execution only: a relaxed arrive
    // (a releasing one waits for this CTA's own global stores, measured 0.6 us per launch).
    if (!cl_waited) cluster_wait();
    cluster_arrive_relaxed();
    cluster_wait();
  }
  if (threadIdx.x == 0) trace_stamp(args, 5, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace apex
