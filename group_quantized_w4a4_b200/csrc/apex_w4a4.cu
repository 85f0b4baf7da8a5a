// apex_w4a4.cu -- host side of the C ABI declared in include/apex_w4a4.h: argument
// validation, TMA descriptor encoding, tile/split selection and kernel launches.
// All device code lives in the headers included below (one translation unit, so the
// library-wide device status word needs no separate device linking).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "apex_w4a4.h"
#include "dual.cuh"
#include "gemm.cuh"
#include "gemm_f8.cuh"
#include "ptx.cuh"
#include "quantize.cuh"

namespace {

using apex::GemmArgs;
using apex::GemmCfg;

uint64_t g_wait_limit_ns = 2000000000ull;
thread_local int t_withhold = -1;
thread_local int t_partials_split = 0;
thread_local unsigned long long* t_trace = nullptr;
thread_local int t_trace_ctas = 0;
thread_local int t_trace_steps = 0;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

apex_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return APEX_OK;
  return APEX_ERR_CUDA;
}

// ------------------------------------------------------------------ device properties

struct DevInfo {
  int sms = 0;
};

DevInfo dev_info() {
  static std::mutex mu;
  static DevInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DevInfo{148};
  std::lock_guard<std::mutex> lk(mu);
  if (!have[dev]) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
    cache[dev].sms = sms;
    have[dev] = true;
  }
  return cache[dev];
}

// ------------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a packed int4 matrix [rows][K/2] bytes; box = 128 bytes (two 128-wide
// K-groups) x box_rows rows, 128-byte swizzle; out-of-range rows and columns read as zeros.
bool make_packed_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over expanded activations [rows][K] bytes (16*q per element); box = 128 bytes
// (one 128-wide K-group) x box_rows rows, 128-byte swizzle: it lands in shared memory in the
// tensor core's K-major operand layout.
bool make_expanded_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map over fp16 [rows][cols] (the outlier dual path's compact operands); box = 64
// halves (128 bytes) x box_rows rows, 128-byte swizzle, zeros outside.
bool make_f16_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ GEMM planning

struct Plan {
  int bt = 128;
  int tiles_n = 0, tiles_m = 0, T = 0;
  int S = 0;        // K-stages (pairs of groups) per tile
  int P = 0;        // persistent CTAs
  int streamk = 0;  // stream-K partition (needs workspace) or whole tiles round-robin
  int cluster = 1;  // >1: each tile split over this many CTAs of one thread-block cluster
};

int pick_bt(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

// One persistent CTA per SM.  Whole tiles when there are at least 4 per SM (the last,
// partial round costs little); otherwise stream-K, so every SM streams the same bytes.
// sms_override > 0 plans for that many SMs instead of the current device's (plan tests).
Plan make_plan(int64_t M, int64_t N, int64_t K, bool allow_streamk, int sms_override = 0) {
  Plan p;
  p.bt = pick_bt(M);
  p.tiles_n = (int)((N + 127) / 128);
  p.tiles_m = (int)((M + p.bt - 1) / p.bt);
  p.T = p.tiles_n * p.tiles_m;
  const int G = (int)(K / 128);
  const int kps = apex::stage_groups(p.bt);
  p.S = (G + kps - 1) / kps;
  const int sms = sms_override > 0 ? sms_override : dev_info().sms;
  if (!allow_streamk || p.T >= 4 * sms) {
    p.streamk = 0;
    p.P = p.T < sms ? p.T : sms;
  } else {
    p.streamk = 1;
    const long long units = (long long)p.T * p.S;
    // With at least two CTAs per tile, split every tile the same number of ways: each CTA
    // then holds one piece of one tile and finishes with a single hand-off, instead of
    // stream-K's pieces of two tiles (a few SMs idle, but the split-K tail halves).
    const int per_tile = sms / p.T;
    const long long want = per_tile >= 2 ? (long long)per_tile * p.T : sms;
    p.P = units < want ? (int)units : (int)want;
    if ((long long)p.P * units >= (1ll << 31)) {   // the device partition math is 32-bit
      p.streamk = 0;
      p.P = p.T < sms ? p.T : sms;
    } else if (per_tile >= 2 && per_tile <= apex::max_cluster(p.bt) && p.S >= per_tile &&
               p.P == per_tile * p.T) {
      // each tile's CTAs as one cluster: the parts are added in the owner's shared memory
      p.cluster = per_tile;
    }
  }
  return p;
}

size_t counters_bytes(const Plan& p) { return (((size_t)p.T * 4) + 255) & ~(size_t)255; }

size_t workspace_for(const Plan& p) {
  if (!p.streamk) return 0;
  return counters_bytes(p) + (size_t)p.P * (size_t)p.bt * 128 * 4;
}

apex_status_t check_gemm_args(int64_t M, int64_t N, int64_t K, int32_t ga, int32_t gw) {
  if (M <= 0 || N <= 0 || K <= 0) return APEX_ERR_INVALID_ARG;
  if (ga <= 0 || gw <= 0 || K % ga || K % gw) return APEX_ERR_INVALID_ARG;
  if (ga != 128) return APEX_ERR_UNSUPPORTED;
  if (gw % 128) return APEX_ERR_UNSUPPORTED;
  if (K % 128) return APEX_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return APEX_ERR_UNSUPPORTED;
  return APEX_OK;
}

struct Maps {
  CUtensorMap w, a;
};

// Every kernel is launched as a programmatic dependent of the previous work in the stream,
// so its launch and prologue overlap that work's tail (each kernel waits for the previous
// grid before its first global access).
// cluster > 1: consecutive CTAs form thread-block clusters of that size.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                          cudaStream_t s, unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = cluster;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t s, Args... args) {
  return launch_pdl_cl(kern, grid, block, smem, s, 1u, args...);
}

template <int BT, int MODE, bool QOUT>
apex_status_t launch_bt(const Plan& p, const Maps& m, GemmArgs a, cudaStream_t s) {
  using C = GemmCfg<BT, MODE, QOUT>;
  auto kern = apex::w4a4_gemm_kernel<BT, MODE, QOUT>;
  static thread_local int attr_dev = -1;   // the attribute is per device; set it once each
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return APEX_ERR_CUDA;
  if (attr_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return APEX_ERR_CUDA;
    attr_dev = dev;
  }
  if (a.cluster > 1) {
    // Clusters only pay when all of them are resident at once (one CTA per SM); otherwise
    // the parts go through global memory.  The answer is cached per device and size.
    static thread_local int occ_dev = -1, occ_size = 0, occ_clusters = 0;
    if (occ_dev != dev || occ_size != a.cluster) {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3((unsigned)p.P);
      cfg.blockDim = dim3(C::THREADS);
      cfg.dynamicSmemBytes = (size_t)C::SMEM;
      cudaLaunchAttribute at{};
      at.id = cudaLaunchAttributeClusterDimension;
      at.val.clusterDim.x = (unsigned)a.cluster;
      at.val.clusterDim.y = 1;
      at.val.clusterDim.z = 1;
      cfg.attrs = &at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
      }
      occ_dev = dev;
      occ_size = a.cluster;
      occ_clusters = n;
    }
    if ((long long)occ_clusters * a.cluster < p.P) a.cluster = 1;
  }
  return cuda_status(launch_pdl_cl(kern, (unsigned)p.P, C::THREADS, (size_t)C::SMEM, s,
                                   (unsigned)a.cluster, m.w, m.a, a));
}

template <int MODE, bool QOUT>
apex_status_t launch_gemm_q(const Plan& p, const Maps& m, const GemmArgs& a, cudaStream_t s) {
  switch (p.bt) {
    case 16: return launch_bt<16, MODE, QOUT>(p, m, a, s);
    case 32: return launch_bt<32, MODE, QOUT>(p, m, a, s);
    case 64: return launch_bt<64, MODE, QOUT>(p, m, a, s);
    default: return launch_bt<128, MODE, QOUT>(p, m, a, s);
  }
}

// The kernel with the quantized output when the arguments ask for one.
template <int MODE>
apex_status_t launch_gemm(const Plan& p, const Maps& m, const GemmArgs& a, cudaStream_t s) {
  if constexpr (MODE != apex::MODE_DUMP) {
    if (a.qout != nullptr) return launch_gemm_q<MODE, true>(p, m, a, s);
  }
  return launch_gemm_q<MODE, false>(p, m, a, s);
}

// Fills the fields every mode shares.
GemmArgs base_args(const Plan& p, int64_t M, int64_t N, int64_t K, int32_t gw,
                   const void* a_scales, const void* w_scales, void* y) {
  GemmArgs a{};
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.gw = gw;
  a.G = (int)(K / 128);
  a.Gw = (int)(K / gw);
  {
    const int gpg = gw / 128;
    a.gpg_shift = (gpg & (gpg - 1)) == 0 ? __builtin_ctz((unsigned)gpg) : -1;
  }
  a.tiles_n = p.tiles_n;
  a.tiles_m = p.tiles_m;
  a.T = p.T;
  a.S = p.S;
  a.kps = apex::stage_groups(p.bt);
  a.TS = p.streamk ? p.T * p.S : 0;
  a.P = p.P;
  a.streamk = p.streamk;
  a.cluster = p.cluster;
  // Scales are fetched in 16-byte blocks of 8 groups when rows are 16-byte strided.
  a.sa_vec = a.G % 8 == 0 && a_scales && aligned(a_scales, 16);
  a.sw_vec = gw == 128 && a.G % 8 == 0 && w_scales && aligned(w_scales, 16);
  a.sa = static_cast<const __half*>(a_scales);
  a.sw = static_cast<const __half*>(w_scales);
  a.y = static_cast<__half*>(y);
  a.wait_ns = g_wait_limit_ns;
  a.withhold = -1;
  return a;
}

void attach_workspace(const Plan& p, GemmArgs& a, void* ws) {
  if (!p.streamk) return;
  a.counters = static_cast<unsigned*>(ws);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + counters_bytes(p));
}

// Units (row, group) each half-warp of the 128-wide-group quantizer takes per round once a
// batch is large enough that the loads in flight, not the per-unit latency, set its time;
// such batches also take the fast per-value path (measured: it loses ~0.1 us on a 16-token
// batch, where one short chain per thread is the whole time, and wins 10-25 % from 512 on).
constexpr int kQuantUnitsPerRound = 2;
constexpr int64_t kQuantBatchMinUnits = 1 << 15;

template <int CH, int FORM, int UPT, bool FAST = true>
cudaError_t quantize_launch_t(int64_t units, cudaStream_t s, const __half* xh, int64_t rows,
                              int64_t K, int32_t group, uint8_t* pk, __half* sc, int g_shift) {
  // 128-thread blocks: one fits on an SM next to a GEMM CTA (registers), so the GEMM that
  // follows can start its prologue on every SM while the quantizer still runs
  const int threads = 128;
  const int64_t warps_needed = (units + 2 * UPT - 1) / (2 * UPT);
  int64_t blocks = (warps_needed * 32 + threads - 1) / threads;
  const int64_t cap = (int64_t)dev_info().sms * 32;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_pdl(apex::quantize_pack_kernel<CH, FORM, UPT, FAST>, (unsigned)blocks, threads,
                    0, s, xh, rows, K, group, pk, sc, g_shift);
}

template <int FORM>
cudaError_t quantize_launch_g128(int64_t units, cudaStream_t s, const __half* xh, int64_t rows,
                                 int64_t K, uint8_t* pk, __half* sc, int g_shift) {
  if (units >= kQuantBatchMinUnits)
    return quantize_launch_t<1, FORM, kQuantUnitsPerRound>(units, s, xh, rows, K, 128, pk, sc,
                                                           g_shift);
  return quantize_launch_t<1, FORM, 1, false>(units, s, xh, rows, K, 128, pk, sc, g_shift);
}

apex_status_t quantize_launch(const void* x, int64_t rows, int64_t K, int32_t group, void* packed,
                              void* scales, void* stream, bool expanded = false,
                              bool e4m3 = false) {
  if (!x || !packed || !scales) return APEX_ERR_INVALID_ARG;
  if (rows <= 0 || K <= 0 || group <= 0 || K % group || group % 128) return APEX_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(packed, (expanded || e4m3) ? 8 : 4) || !aligned(scales, 2))
    return APEX_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t units = rows * (K / group);
  if (units >= (1ll << 31)) return APEX_ERR_UNSUPPORTED;   // the kernel indexes units in 32 bits
  const int64_t gpr = K / group;                             // groups per row
  const int g_shift = (gpr & (gpr - 1)) == 0 ? __builtin_ctzll((unsigned long long)gpr) : -1;
  const __half* xh = static_cast<const __half*>(x);
  uint8_t* pk = static_cast<uint8_t*>(packed);
  __half* sc = static_cast<__half*>(scales);
  cudaError_t e;
  if (e4m3) {
    if (group == 128)
      e = quantize_launch_g128<apex::FORM_E4M3>(units, s, xh, rows, K, pk, sc, g_shift);
    else if (group == 512)
      e = quantize_launch_t<4, apex::FORM_E4M3, 1>(units, s, xh, rows, K, group, pk, sc, g_shift);
    else
      e = quantize_launch_t<0, apex::FORM_E4M3, 1>(units, s, xh, rows, K, group, pk, sc, g_shift);
  } else if (expanded) {
    if (group != 128) return APEX_ERR_UNSUPPORTED;
    e = quantize_launch_g128<apex::FORM_EXPANDED>(units, s, xh, rows, K, pk, sc, g_shift);
  } else if (group == 128) {
    e = quantize_launch_g128<apex::FORM_PACKED>(units, s, xh, rows, K, pk, sc, g_shift);
  } else if (group == 256) {
    e = quantize_launch_t<2, apex::FORM_PACKED, 1>(units, s, xh, rows, K, group, pk, sc, g_shift);
  } else if (group == 512) {
    e = quantize_launch_t<4, apex::FORM_PACKED, 1>(units, s, xh, rows, K, group, pk, sc, g_shift);
  } else {
    e = quantize_launch_t<0, apex::FORM_PACKED, 1>(units, s, xh, rows, K, group, pk, sc, g_shift);
  }
  if (e != cudaSuccess) return APEX_ERR_CUDA;
  return cuda_status(cudaPeekAtLastError());
}

// apex_w4a4_linear: the activation form the quantizer writes for a batch of M tokens
// (expanded from 128 tokens on, where activation bytes are small next to the math).
constexpr int64_t kLinearExpandedMinM = 128;

size_t linear_act_bytes(int64_t M, int64_t K) {   // quantized activations + their scales
  const int64_t per_row = M >= kLinearExpandedMinM ? K : K / 2;
  const size_t a = (((size_t)M * (size_t)per_row) + 255) & ~(size_t)255;
  const size_t sc = (((size_t)M * (size_t)(K / 128) * 2) + 255) & ~(size_t)255;
  return a + sc;
}

// The quantized output of a GEMM (all null: none).
struct QuantOut {
  void* q = nullptr;        // packed [M][N/2] or expanded [M][N]
  void* scales = nullptr;   // fp16 [M][N/128]
  bool expanded = false;
};

// Everything apex_w4a4_gemm and its variants share: argument checks, plan, launch.
// y may be null when a quantized output is requested.
apex_status_t gemm_entry(bool a_expanded, int64_t M, int64_t N, int64_t K, int32_t group_a,
                         int32_t group_w, const void* a_q, const void* a_scales,
                         const void* w_packed, const void* w_scales, void* y_f16,
                         const QuantOut& qo, void* workspace, size_t workspace_bytes,
                         void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!a_q || !a_scales || !w_packed || !w_scales) return APEX_ERR_INVALID_ARG;
  if (!y_f16 && !qo.q) return APEX_ERR_INVALID_ARG;
  if (qo.q && !qo.scales) return APEX_ERR_INVALID_ARG;
  if (qo.q && N % 128) return APEX_ERR_UNSUPPORTED;   // the output's groups are whole tiles
  if (!aligned(a_q, 16) || !aligned(w_packed, 16) || !aligned(a_scales, 2) ||
      !aligned(w_scales, 2) || (y_f16 && !aligned(y_f16, 2)) ||
      (qo.q && (!aligned(qo.q, 16) || !aligned(qo.scales, 2))) ||
      (workspace && !aligned(workspace, 256)))
    return APEX_ERR_ALIGNMENT;

  Plan p = make_plan(M, N, K, true);
  // Without a large enough workspace, whole tiles only.
  if (p.streamk && (!workspace || workspace_for(p) > workspace_bytes)) p = make_plan(M, N, K, false);
  GemmArgs a = base_args(p, M, N, K, group_w, a_scales, w_scales, y_f16);
  a.qout = static_cast<uint8_t*>(qo.q);
  a.qscale = static_cast<__half*>(qo.scales);
  a.qexp = qo.expanded ? 1 : 0;
  attach_workspace(p, a, workspace);
  a.withhold = t_withhold;
  t_withhold = -1;
  a.trace = t_trace;
  a.trace_ctas = t_trace_ctas;
  a.trace_steps = t_trace_steps;
  t_trace = nullptr;

  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_packed_map(&maps.w, w_packed, N, K, 128)) return APEX_ERR_CUDA;
  if (a_expanded ? !make_expanded_map(&maps.a, a_q, M, K, p.bt)
                 : !make_packed_map(&maps.a, a_q, M, K, p.bt))
    return APEX_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return a_expanded ? launch_gemm<apex::MODE_AQ8>(p, maps, a, s)
                    : launch_gemm<apex::MODE_PACKED>(p, maps, a, s);
}

// ------------------------------------------------------------------ the E4M3-carrier GEMM

struct F8Plan {
  int tiles_m = 0, tiles_n = 0, T = 0, P = 0;
};

F8Plan make_f8_plan(int64_t M, int64_t N, int sms_override = 0) {
  F8Plan p;
  p.tiles_m = (int)((M + 127) / 128);
  p.tiles_n = (int)((N + 255) / 256);
  p.T = p.tiles_m * p.tiles_n;
  const int sms = sms_override > 0 ? sms_override : dev_info().sms;
  p.P = p.T < sms ? p.T : sms;
  return p;
}

#ifndef APEX_F8_EPI_WARPS
#define APEX_F8_EPI_WARPS 8
#endif

template <int MODE, bool DUAL = false, bool QOUT = false>
apex_status_t launch_f8(const F8Plan& p, const CUtensorMap& ma, const CUtensorMap& mb,
                        const apex::F8Args& a, cudaStream_t s, const CUtensorMap& mxo_,
                        const CUtensorMap& mwo_) {
  using C = apex::F8Cfg<APEX_F8_EPI_WARPS>;
  auto kern = apex::w4a4_gemm_f8_kernel<MODE, APEX_F8_EPI_WARPS, DUAL, QOUT>;
  static thread_local int attr_dev = -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return APEX_ERR_CUDA;
  if (attr_dev != dev) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
        cudaSuccess)
      return APEX_ERR_CUDA;
    attr_dev = dev;
  }
  // without the outlier dual path the outlier maps are never read: the operand maps stand in
  const CUtensorMap& mxo = a.NO > 0 ? mxo_ : ma;
  const CUtensorMap& mwo = a.NO > 0 ? mwo_ : mb;
  return cuda_status(
      launch_pdl(kern, (unsigned)p.P, C::THREADS, (size_t)C::SMEM, s, ma, mb, mxo, mwo, a));
}

// The shared part of apex_w4a4_gemm_fp8 and the partials export: checks, plan, maps.
apex_status_t f8_setup(int64_t M, int64_t N, int64_t K, int32_t group_w, const void* a_codes,
                       const void* w_codes, F8Plan& p, apex::F8Args& a, CUtensorMap& ma,
                       CUtensorMap& mb) {
  if (!a_codes || !w_codes) return APEX_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(w_codes, 16)) return APEX_ERR_ALIGNMENT;
  p = make_f8_plan(M, N);
  memset(&a, 0, sizeof(a));
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.G = (int)(K / 128);
  a.Gw = (int)(K / group_w);
  a.gpg = group_w / 128;
  a.gpg_shift = (a.gpg & (a.gpg - 1)) == 0 ? __builtin_ctz((unsigned)a.gpg) : -1;
  a.tiles_m = p.tiles_m;
  a.tiles_n = p.tiles_n;
  a.T = p.T;
  a.P = p.P;
  a.wait_ns = g_wait_limit_ns;
  memset(&ma, 0, sizeof(ma));
  memset(&mb, 0, sizeof(mb));
  if (!make_expanded_map(&ma, a_codes, M, K, 128) || !make_expanded_map(&mb, w_codes, N, K, 256))
    return APEX_ERR_CUDA;
  return APEX_OK;
}

}  // namespace

extern "C" {

apex_status_t apex_quantize_act_int4_fp8(const void* x_f16, int64_t M, int64_t K,
                                         int32_t group_a, void* x_codes, void* x_scales_f16,
                                         void* stream) {
  if (group_a != 128 && group_a > 0 && K % group_a == 0 && group_a % 128 == 0)
    return APEX_ERR_UNSUPPORTED;
  return quantize_launch(x_f16, M, K, group_a, x_codes, x_scales_f16, stream, false, true);
}

apex_status_t apex_pack_weights_int4_fp8(const void* w_f16, int64_t N, int64_t K,
                                         int32_t group_w, void* w_codes, void* w_scales_f16,
                                         void* stream) {
  return quantize_launch(w_f16, N, K, group_w, w_codes, w_scales_f16, stream, false, true);
}

apex_status_t apex_unpack_int4_fp8(const void* packed, int64_t rows, int64_t K, void* codes,
                                   void* stream) {
  if (!packed || !codes) return APEX_ERR_INVALID_ARG;
  if (rows <= 0 || K <= 0 || K % 16) return APEX_ERR_INVALID_ARG;
  if (!aligned(packed, 8) || !aligned(codes, 16)) return APEX_ERR_ALIGNMENT;
  const int64_t words = rows * (K / 16);   // 8 packed bytes -> 16 codes each
  int64_t blocks = (words + 255) / 256;
  const int64_t cap = (int64_t)dev_info().sms * 8;
  if (blocks > cap) blocks = cap;
  cudaError_t e = launch_pdl(apex::unpack_e4m3_kernel, (unsigned)blocks, 256, 0,
                             static_cast<cudaStream_t>(stream),
                             static_cast<const uint8_t*>(packed), words,
                             static_cast<uint8_t*>(codes));
  if (e != cudaSuccess) return APEX_ERR_CUDA;
  return cuda_status(cudaPeekAtLastError());
}

apex_status_t apex_w4a4_gemm_fp8(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                 int32_t group_w, const void* a_codes, const void* a_scales,
                                 const void* w_codes, const void* w_scales, void* y_f16,
                                 void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!a_scales || !w_scales || !y_f16) return APEX_ERR_INVALID_ARG;
  if (!aligned(a_scales, 2) || !aligned(w_scales, 2) || !aligned(y_f16, 2))
    return APEX_ERR_ALIGNMENT;
  F8Plan p;
  apex::F8Args a;
  CUtensorMap ma, mb;
  st = f8_setup(M, N, K, group_w, a_codes, w_codes, p, a, ma, mb);
  if (st != APEX_OK) return st;
  a.sa = static_cast<const __half*>(a_scales);
  a.sw = static_cast<const __half*>(w_scales);
  a.y = static_cast<__half*>(y_f16);
  a.sa_vec = a.G % 8 == 0 && aligned(a_scales, 16);
  a.sw_vec = group_w == 128 && a.G % 8 == 0 && aligned(w_scales, 16);
  a.y_vec = N % 8 == 0 && aligned(y_f16, 16);
  // per-channel weight groups: the weight scale factors out of the K sum
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return group_w == K ? launch_f8<apex::F8_PER_CHANNEL>(p, ma, mb, a, s, ma, mb)
                      : launch_f8<apex::F8_GROUPED>(p, ma, mb, a, s, ma, mb);
}

apex_status_t apex_w4a4_gemm_fp8_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                       int32_t group_w, const void* a_codes,
                                       const void* a_scales, const void* w_codes,
                                       const void* w_scales, void* y_f16, void* yq_codes,
                                       void* yq_scales, void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!a_scales || !w_scales || !yq_codes || !yq_scales) return APEX_ERR_INVALID_ARG;
  if (N % 128) return APEX_ERR_UNSUPPORTED;   // every 128 outputs are one next-layer group
  if (!aligned(a_scales, 2) || !aligned(w_scales, 2) || (y_f16 && !aligned(y_f16, 2)) ||
      !aligned(yq_codes, 16) || !aligned(yq_scales, 2))
    return APEX_ERR_ALIGNMENT;
  F8Plan p;
  apex::F8Args a;
  CUtensorMap ma, mb;
  st = f8_setup(M, N, K, group_w, a_codes, w_codes, p, a, ma, mb);
  if (st != APEX_OK) return st;
  a.sa = static_cast<const __half*>(a_scales);
  a.sw = static_cast<const __half*>(w_scales);
  a.y = static_cast<__half*>(y_f16);
  a.qout = static_cast<uint8_t*>(yq_codes);
  a.qscale = static_cast<__half*>(yq_scales);
  a.sa_vec = a.G % 8 == 0 && aligned(a_scales, 16);
  a.sw_vec = group_w == 128 && a.G % 8 == 0 && aligned(w_scales, 16);
  a.y_vec = y_f16 && N % 8 == 0 && aligned(y_f16, 16);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return group_w == K ? launch_f8<apex::F8_PER_CHANNEL, false, true>(p, ma, mb, a, s, ma, mb)
                      : launch_f8<apex::F8_GROUPED, false, true>(p, ma, mb, a, s, ma, mb);
}

apex_status_t apex_w4a4_group_partials_fp8(int64_t M, int64_t N, int64_t K, const void* a_codes,
                                           const void* w_codes, int32_t* partials_i32,
                                           void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, 128, 128);
  if (st != APEX_OK) return st;
  if (!partials_i32) return APEX_ERR_INVALID_ARG;
  if (!aligned(partials_i32, 4)) return APEX_ERR_ALIGNMENT;
  F8Plan p;
  apex::F8Args a;
  CUtensorMap ma, mb;
  st = f8_setup(M, N, K, 128, a_codes, w_codes, p, a, ma, mb);
  if (st != APEX_OK) return st;
  a.dump = partials_i32;
  return launch_f8<apex::F8_DUMP>(p, ma, mb, a, static_cast<cudaStream_t>(stream), ma, mb);
}

apex_status_t apex_pack_weights_int4(const void* w_f16, int64_t N, int64_t K, int32_t group_w,
                                     void* w_packed_u8, void* w_scales_f16, void* stream) {
  return quantize_launch(w_f16, N, K, group_w, w_packed_u8, w_scales_f16, stream);
}

apex_status_t apex_quantize_act_int4(const void* x_f16, int64_t M, int64_t K, int32_t group_a,
                                     void* x_packed_u8, void* x_scales_f16, void* stream) {
  return quantize_launch(x_f16, M, K, group_a, x_packed_u8, x_scales_f16, stream);
}

apex_status_t apex_quantize_act_int4_expanded(const void* x_f16, int64_t M, int64_t K,
                                              int32_t group_a, void* x_q8, void* x_scales_f16,
                                              void* stream) {
  return quantize_launch(x_f16, M, K, group_a, x_q8, x_scales_f16, stream, true);
}

apex_status_t apex_w4a4_gemm_expanded(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                      int32_t group_w, const void* a_q8, const void* a_scales,
                                      const void* w_packed, const void* w_scales, void* y_f16,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (!y_f16) return APEX_ERR_INVALID_ARG;
  return gemm_entry(true, M, N, K, group_a, group_w, a_q8, a_scales, w_packed, w_scales, y_f16,
                    QuantOut{}, workspace, workspace_bytes, stream);
}

apex_status_t apex_w4a4_gemm_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                   int32_t group_w, const void* a_packed, const void* a_scales,
                                   const void* w_packed, const void* w_scales, void* y_f16,
                                   void* yq, void* yq_scales, int32_t yq_expanded,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  QuantOut qo;
  qo.q = yq;
  qo.scales = yq_scales;
  qo.expanded = yq_expanded != 0;
  if (!yq) return APEX_ERR_INVALID_ARG;
  return gemm_entry(false, M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales,
                    y_f16, qo, workspace, workspace_bytes, stream);
}

apex_status_t apex_w4a4_gemm_expanded_quant(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                            int32_t group_w, const void* a_q8,
                                            const void* a_scales, const void* w_packed,
                                            const void* w_scales, void* y_f16, void* yq,
                                            void* yq_scales, int32_t yq_expanded,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  QuantOut qo;
  qo.q = yq;
  qo.scales = yq_scales;
  qo.expanded = yq_expanded != 0;
  if (!yq) return APEX_ERR_INVALID_ARG;
  return gemm_entry(true, M, N, K, group_a, group_w, a_q8, a_scales, w_packed, w_scales, y_f16,
                    qo, workspace, workspace_bytes, stream);
}

size_t apex_w4a4_linear_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                       int32_t group_w) {
  if (check_gemm_args(M, N, K, group_a, group_w) != APEX_OK) return 0;
  return linear_act_bytes(M, K) + workspace_for(make_plan(M, N, K, true));
}

apex_status_t apex_w4a4_linear(int64_t M, int64_t N, int64_t K, int32_t group_a,
                               int32_t group_w, const void* x_f16, const void* w_packed,
                               const void* w_scales, void* y_f16, void* workspace,
                               size_t workspace_bytes, void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!x_f16 || !w_packed || !w_scales || !y_f16) return APEX_ERR_INVALID_ARG;
  if (!aligned(x_f16, 16) || !aligned(w_packed, 16) || !aligned(w_scales, 2) ||
      !aligned(y_f16, 2) || (workspace && !aligned(workspace, 256)))
    return APEX_ERR_ALIGNMENT;
  const size_t act = linear_act_bytes(M, K);
  if (!workspace || workspace_bytes < act) return APEX_ERR_INVALID_ARG;
  const bool expanded = M >= kLinearExpandedMinM;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* a_q = ws;
  void* a_sc = ws + ((((size_t)M * (size_t)(expanded ? K : K / 2)) + 255) & ~(size_t)255);
  st = quantize_launch(x_f16, M, K, 128, a_q, a_sc, stream, expanded);
  if (st != APEX_OK) return st;
  return expanded ? apex_w4a4_gemm_expanded(M, N, K, group_a, group_w, a_q, a_sc, w_packed,
                                            w_scales, y_f16, ws + act, workspace_bytes - act,
                                            stream)
                  : apex_w4a4_gemm(M, N, K, group_a, group_w, a_q, a_sc, w_packed, w_scales,
                                   y_f16, ws + act, workspace_bytes - act, stream);
}

size_t apex_w4a4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                     int32_t group_w) {
  if (check_gemm_args(M, N, K, group_a, group_w) != APEX_OK) return 0;
  return workspace_for(make_plan(M, N, K, true));
}

apex_status_t apex_w4a4_gemm(int64_t M, int64_t N, int64_t K, int32_t group_a, int32_t group_w,
                             const void* a_packed, const void* a_scales, const void* w_packed,
                             const void* w_scales, void* y_f16, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!y_f16) return APEX_ERR_INVALID_ARG;
  return gemm_entry(false, M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales,
                    y_f16, QuantOut{}, workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ allocation-free GEMM
//
// For callers that may not allocate device memory while they run: serving runtimes that
// plan every device byte ahead of time and hand out no scratch, plugin hosts whose
// allocator is off limits to the plugin, and code paths that must not pay for
// cudaMalloc/cudaFree (which can stall or synchronize the whole device).  The split-K
// scratch lives in this fixed, library-owned device array instead: every GPU that loads
// the library keeps APEX_STATIC_SCRATCH_BYTES reserved until the process exits.
static __device__ __align__(256) uint8_t g_static_scratch[APEX_STATIC_SCRATCH_BYTES];

namespace {

// Device address of g_static_scratch, looked up once per device (with that device current)
// on the first call there, and kept until the process exits (a device reset afterwards is
// not supported).  The array's host-side name is only a handle, never an address.
apex_status_t static_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return APEX_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return APEX_ERR_CUDA;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return APEX_OK;
}

}  // namespace

apex_status_t apex_w4a4_gemm_noalloc(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                     int32_t group_w, const void* a_packed, const void* a_scales,
                                     const void* w_packed, const void* w_scales, void* y_f16,
                                     void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!a_packed || !a_scales || !w_packed || !w_scales || !y_f16) return APEX_ERR_INVALID_ARG;
  if (!aligned(a_packed, 16) || !aligned(w_packed, 16) || !aligned(a_scales, 2) ||
      !aligned(w_scales, 2) || !aligned(y_f16, 2))
    return APEX_ERR_ALIGNMENT;

  Plan p = make_plan(M, N, K, true);
  // The problem's stream-K scratch must fit the fixed array; larger problems are refused.
  if (workspace_for(p) > (size_t)APEX_STATIC_SCRATCH_BYTES) return APEX_ERR_UNSUPPORTED;
  GemmArgs a = base_args(p, M, N, K, group_w, a_scales, w_scales, y_f16);
  a.withhold = t_withhold;   // test hook, as in apex_w4a4_gemm
  t_withhold = -1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.streamk) {
    void* scratch = nullptr;
    st = static_scratch_ptr(&scratch);
    if (st != APEX_OK) return st;
    // The array keeps whatever the previous call left: the arrival counters start at zero.
    if (cudaMemsetAsync(scratch, 0, counters_bytes(p), s) != cudaSuccess) return APEX_ERR_CUDA;
    attach_workspace(p, a, scratch);
  }
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_packed_map(&maps.w, w_packed, N, K, 128) ||
      !make_packed_map(&maps.a, a_packed, M, K, p.bt))
    return APEX_ERR_CUDA;
  return launch_gemm<apex::MODE_PACKED>(p, maps, a, s);
}

apex_status_t apex_w4a4_group_partials(int64_t M, int64_t N, int64_t K, const void* a_packed,
                                       const void* w_packed, int32_t* partials_i32,
                                       void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, 128, 128);
  if (st != APEX_OK) return st;
  if (!a_packed || !w_packed || !partials_i32) return APEX_ERR_INVALID_ARG;
  if (!aligned(a_packed, 16) || !aligned(w_packed, 16) || !aligned(partials_i32, 4))
    return APEX_ERR_ALIGNMENT;
  // The work plan: whole tiles, or (test hook) the split plan apex_w4a4_gemm takes with a
  // workspace -- each (tile, K-group) is still handled by exactly one CTA, which stores its
  // partial, so no scratch is needed and the split parts are never added.
  Plan p = make_plan(M, N, K, t_partials_split != 0);
  t_partials_split = 0;
  GemmArgs a = base_args(p, M, N, K, 128, nullptr, nullptr, nullptr);
  a.cluster = 1;
  a.dump = partials_i32;
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if (!make_packed_map(&maps.w, w_packed, N, K, 128) ||
      !make_packed_map(&maps.a, a_packed, M, K, p.bt))
    return APEX_ERR_CUDA;
  return launch_gemm<apex::MODE_DUMP>(p, maps, a, static_cast<cudaStream_t>(stream));
}

apex_status_t apex_get_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return APEX_ERR_CUDA;
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, apex::g_device_status, sizeof(v)) != cudaSuccess)
    return APEX_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(apex::g_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return APEX_ERR_CUDA;
  if (v & apex::DEV_TIMEOUT) return APEX_ERR_TIMEOUT;
  return APEX_OK;
}

void apex_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns = ns ? ns : 1; }

apex_status_t apex_debug_gemm_plan(int64_t M, int64_t N, int64_t K, int32_t sms,
                                   int32_t with_workspace, int32_t *plan) {
  if (!plan || sms <= 0) return APEX_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 || M > INT32_MAX || N > INT32_MAX ||
      K > INT32_MAX)
    return APEX_ERR_INVALID_ARG;
  const Plan p = make_plan(M, N, K, with_workspace != 0, sms);
  plan[0] = p.bt;
  plan[1] = p.T;
  plan[2] = p.S;
  plan[3] = p.P;
  plan[4] = p.streamk;
  plan[5] = p.cluster;
  return APEX_OK;
}

int32_t apex_select_weight_group(int64_t M, int64_t N, int64_t K, double rho,
                                 double ridge_ops_per_byte) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 128 || !(rho > 0.0) || !(ridge_ops_per_byte > 0.0))
    return 0;
  // Below the ridge the weight stream bounds the GEMM and the dequantisation hides behind
  // it: keep the finest groups.
  const double bytes = (double)M * K / 2 + (double)N * K / 2 + 2.0 * M * (K / 128) +
                       2.0 * N * (K / 128) + 2.0 * M * N;
  const double intensity = 2.0 * M * N * K / bytes;
  if (intensity < ridge_ops_per_byte) return 128;
  // Above it, per output and per 128-wide K-group the tensor cores do 2*128 operations and
  // the CUDA cores the dequantisation: with 128-wide weight groups one fp32 product of the
  // two scales and one fma (4 operations), with one weight scale per row only the fma (2;
  // the scale is applied once after the sum).  At rho times the CUDA-core rate, the
  // dequantisation takes d * rho / 256 of the tensor time; keep 128-wide groups while that
  // is at most half.
  if (4.0 * rho / 256.0 <= 0.5) return 128;
  return (int32_t)K;
}

void apex_debug_withhold_step(int32_t step) { t_withhold = step; }

void apex_debug_partials_split(int32_t on) { t_partials_split = on ? 1 : 0; }

void apex_debug_trace_next_gemm(uint64_t* trace, int32_t ctas, int32_t steps) {
  t_trace = reinterpret_cast<unsigned long long*>(trace);
  t_trace_ctas = ctas;
  t_trace_steps = steps;
}

const char* apex_status_string(apex_status_t status) {
  switch (status) {
    case APEX_OK: return "ok";
    case APEX_ERR_INVALID_ARG: return "invalid argument";
    case APEX_ERR_UNSUPPORTED: return "unsupported configuration";
    case APEX_ERR_ALIGNMENT: return "misaligned pointer";
    case APEX_ERR_CUDA: return "CUDA error";
    case APEX_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------- outlier dual path

namespace {

apex_status_t check_outlier_args(int64_t K, const void* channels, int32_t C, int32_t Cp) {
  if (!channels || C < 1 || C > K || Cp < C || Cp % 64) return APEX_ERR_INVALID_ARG;
  if (!aligned(channels, 4)) return APEX_ERR_ALIGNMENT;
  return APEX_OK;
}

unsigned grid_for(int64_t work, int threads, int per_sm) {
  int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)dev_info().sms * per_sm;
  if (blocks > cap) blocks = cap;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

}  // namespace

extern "C" {

apex_status_t apex_gather_weight_columns(const void* w_f16, int64_t N, int64_t K,
                                         const void* channels, int32_t C, void* w_out_f16,
                                         int32_t Cp, void* stream) {
  if (!w_f16 || !w_out_f16 || N <= 0 || K <= 0) return APEX_ERR_INVALID_ARG;
  apex_status_t st = check_outlier_args(K, channels, C, Cp);
  if (st != APEX_OK) return st;
  if (!aligned(w_f16, 2) || !aligned(w_out_f16, 16)) return APEX_ERR_ALIGNMENT;
  cudaError_t e = launch_pdl(apex::gather_columns_kernel, grid_for(N * (int64_t)Cp, 256, 16), 256,
                             0, static_cast<cudaStream_t>(stream),
                             static_cast<const __half*>(w_f16), N, K,
                             static_cast<const int32_t*>(channels), (int)C,
                             static_cast<__half*>(w_out_f16), (int)Cp);
  if (e != cudaSuccess) return APEX_ERR_CUDA;
  return cuda_status(cudaPeekAtLastError());
}

apex_status_t apex_quantize_act_int4_dual(const void* x_f16, int64_t M, int64_t K,
                                          int32_t group_a, const void* channels, int32_t C,
                                          int32_t form, void* x_q, void* x_scales_f16,
                                          void* x_out_f16, int32_t Cp, void* stream) {
  if (!x_f16 || !x_q || !x_scales_f16 || !x_out_f16) return APEX_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || K % 128) return APEX_ERR_INVALID_ARG;
  if (form < APEX_FORM_PACKED || form > APEX_FORM_FP8) return APEX_ERR_INVALID_ARG;
  if (group_a != 128) return APEX_ERR_UNSUPPORTED;
  apex_status_t st = check_outlier_args(K, channels, C, Cp);
  if (st != APEX_OK) return st;
  if (!aligned(x_f16, 16) || !aligned(x_q, form == APEX_FORM_PACKED ? 4 : 8) ||
      !aligned(x_scales_f16, 2) || !aligned(x_out_f16, 16))
    return APEX_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t G = K / 128;
  if (M * G >= (1ll << 31) || C >= 65536) return APEX_ERR_UNSUPPORTED;   // 32-bit units, 16-bit table
  const int g_shift = (G & (G - 1)) == 0 ? __builtin_ctzll((unsigned long long)G) : -1;
  const size_t tab = apex::dual_table_bytes(K);
  if (tab > 200 * 1024) return APEX_ERR_UNSUPPORTED;
  const unsigned nb = grid_for(((M * G + 1) / 2) * 32, 128, 32);
  const __half* xh = static_cast<const __half*>(x_f16);
  const int32_t* ch = static_cast<const int32_t*>(channels);
  uint8_t* q = static_cast<uint8_t*>(x_q);
  __half* sc = static_cast<__half*>(x_scales_f16);
  __half* xo = static_cast<__half*>(x_out_f16);
  auto run = [&](auto kern) -> cudaError_t {
    if (tab > 48 * 1024) {
      const cudaError_t ea =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tab);
      if (ea != cudaSuccess) return ea;
    }
    return launch_pdl(kern, nb, 128, tab, s, xh, M, K, ch, (int)C, q, sc, xo, (int)Cp, g_shift);
  };
  cudaError_t e;
  if (form == APEX_FORM_FP8)
    e = run(apex::quantize_dual_kernel<apex::FORM_E4M3>);
  else if (form == APEX_FORM_EXPANDED)
    e = run(apex::quantize_dual_kernel<apex::FORM_EXPANDED>);
  else
    e = run(apex::quantize_dual_kernel<apex::FORM_PACKED>);
  if (e != cudaSuccess) return APEX_ERR_CUDA;
  return cuda_status(cudaPeekAtLastError());
}

apex_status_t apex_w4a4_gemm_fp8_dual(int64_t M, int64_t N, int64_t K, int32_t group_a,
                                      int32_t group_w, const void* a_codes,
                                      const void* a_scales, const void* w_codes,
                                      const void* w_scales, const void* x_out_f16,
                                      const void* w_out_f16, int32_t Cp, void* y_f16,
                                      void* stream) {
  apex_status_t st = check_gemm_args(M, N, K, group_a, group_w);
  if (st != APEX_OK) return st;
  if (!a_scales || !w_scales || !y_f16 || !x_out_f16 || !w_out_f16) return APEX_ERR_INVALID_ARG;
  if (Cp < 64 || Cp % 64 || Cp > K) return APEX_ERR_INVALID_ARG;
  if (!aligned(a_scales, 2) || !aligned(w_scales, 2) || !aligned(y_f16, 2) ||
      !aligned(x_out_f16, 16) || !aligned(w_out_f16, 16))
    return APEX_ERR_ALIGNMENT;
  F8Plan p;
  apex::F8Args a;
  CUtensorMap ma, mb, mxo, mwo;
  st = f8_setup(M, N, K, group_w, a_codes, w_codes, p, a, ma, mb);
  if (st != APEX_OK) return st;
  memset(&mxo, 0, sizeof(mxo));
  memset(&mwo, 0, sizeof(mwo));
  if (!make_f16_map(&mxo, x_out_f16, M, Cp, 128) || !make_f16_map(&mwo, w_out_f16, N, Cp, 256))
    return APEX_ERR_CUDA;
  a.sa = static_cast<const __half*>(a_scales);
  a.sw = static_cast<const __half*>(w_scales);
  a.y = static_cast<__half*>(y_f16);
  a.sa_vec = a.G % 8 == 0 && aligned(a_scales, 16);
  a.sw_vec = group_w == 128 && a.G % 8 == 0 && aligned(w_scales, 16);
  a.y_vec = N % 8 == 0 && aligned(y_f16, 16);
  a.NO = Cp / 64;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return group_w == K ? launch_f8<apex::F8_PER_CHANNEL, true>(p, ma, mb, a, s, mxo, mwo)
                      : launch_f8<apex::F8_GROUPED, true>(p, ma, mb, a, s, mxo, mwo);
}

}  // extern "C"
