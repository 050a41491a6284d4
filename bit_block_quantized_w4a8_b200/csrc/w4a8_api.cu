// w4a8_api.cu -- the C ABI of libw4a8.so (declared in include/w4a8.h):
// host-side argument checks, schedule selection, tensor-map encoding and
// kernel launches.  One translation unit: the kernels live in the .cuh
// files included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "gemm.cuh"
#include "gemm_pp.cuh"
#include "gemv.cuh"
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "w4a8.h"

namespace w4a8 {



namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kMaxDevices = 64;

// Budget of the kernels' main-loop waits: 2 s, or a test budget set by
// w4a8_debug_set_wait_budget (0 = every such wait expires at once).
std::atomic<long long> g_wait_budget{-1};
unsigned long long wait_budget() {
  const long long v = g_wait_budget.load(std::memory_order_relaxed);
  return v < 0 ? kWaitLimitNs : (unsigned long long)v;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

int num_sms(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over Xq [M][K] int8 (K contiguous): boxes of 128 bytes of k by
// `rows` tokens, 128-byte swizzle, zero fill past row M.
bool make_act_map(CUtensorMap* map, const int8_t* Xq, int M, int K, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(Xq), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the bf16 output Y [M][N] (N contiguous) for the TMA store
// of a tile: boxes of 128 channels by `rows` tokens, no swizzle; the store
// leaves elements outside [M, N] alone.  Needs N a multiple of 8 (16-byte
// row stride) and Y 16-byte aligned.
bool make_y_map(CUtensorMap* map, uint16_t* Y, int M, int N, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)N * 2};
  cuuint32_t box[2] = {(cuuint32_t)kTileN, (cuuint32_t)rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, Y, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over INT8 weights Wq [N][K] (K contiguous), for the W8A8
// comparison kernel: boxes of 128 bytes of k by 128 channels, 128-byte
// swizzle (the MMA's K-major operand layout), zero fill past channel N.
bool make_w8_map(CUtensorMap* map, const int8_t* Wq, int N, int K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)kTileN};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(Wq), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// -------------------------------------------------- kernel attributes
template <int T, int SS, int AS, int DQG, int MINB, bool PUSH = false, bool W8 = false,
          int V = kVarDefault, bool PAIR = false, bool RTN = false, bool FUSED = false>
cudaError_t ensure_smem_attr() {
  using C = GemmCfg<T, SS, AS, DQG, PUSH, W8, PAIR, FUSED>;
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load(std::memory_order_relaxed)) {
    cudaError_t e = cudaFuncSetAttribute(
        w4a8_gemm_kernel<T, SS, AS, DQG, MINB, PUSH, W8, V, PAIR, RTN, FUSED>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  return cudaSuccess;
}

// ------------------------------------------------------------ schedule
struct Schedule {
  int T = 16, splits = 1, kt_per = 1, n_tiles = 1, m_tiles = 1, ctas = 1;
};

constexpr int kMaxSplits = 8;  // portable thread-block cluster size
constexpr int kRasterBand = 8;  // token tiles per raster band (dense GEMMs)

// Tokens per tile: the smallest MMA N (multiple of 16, up to 256) that
// covers M, so decode shapes do no wasted MMA work beyond 16 tokens.
// (Above 64 tokens the 256-token tile is used: one CTA per SM with a deeper
// ring measured faster than two 128-token CTAs per SM.)
int tile_tokens(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 256; }

// 16-token tiles walking at most this many k tiles use the light ring
// (three CTAs per SM).  W4A8_LIGHT16=0 in the environment turns it off
// (tuning experiments only).
constexpr int kLightMaxKt = 6;
bool light16_enabled() {
  static const bool ok = [] {
    const char* v = getenv("W4A8_LIGHT16");
    return !(v && v[0] == '0');
  }();
  return ok;
}

// The CTA-pair form of the 256-token tile (see use_pair below).
// W4A8_PAIR=0 in the environment turns it off (tuning only).
bool pair_enabled() {
  static const bool enabled = [] {
    const char* v = getenv("W4A8_PAIR");
    return !(v && v[0] == '0');
  }();
  return enabled;
}

// CTAs of one configuration that fit on an SM at once (shared memory and
// TMEM permitting); matches the MINB column of the launch tables below.
int ctas_per_sm(int T, int kt_per, bool w8) {
  if (!w8 && T == 16 && kt_per <= kLightMaxKt && light16_enabled()) return 3;
  return T <= 128 ? 2 : 1;
}

// Split-K factor from a latency/bandwidth model of one launch, in
// microseconds, calibrated on B200 against forced-split timings of the
// decode and 7B/70B-like layer shapes:
//   time = waves * (fill + kt_per * t_tile) + reduction
// - a wave is as many clusters (the splits of one output tile) as the SMs
//   hold at once; a cluster whose size is not a power of two does not tile
//   the SMs of a GPC evenly, so only 92% of the slots count for it;
// - fill is launch, pipeline fill and epilogue (3 us for 16..64-token
//   tiles, 7.4 us for the 256-token tile);
// - t_tile is one k tile's time per CTA: the slower of the CTA's own
//   dequantize + MMA chain (0.27 us for 16 tokens, 0.29 us for 256) and its
//   share of HBM bandwidth (8.7 KB of packed weights per CTA per k tile at
//   6 TB/s sustained); the W8A8 comparison kernel reads 16 KB of weights
//   per k tile through a shallower ring (bytes in flight per CTA bound it:
//   0.35..0.45 us per k tile);
// - the cluster reduction: the push form ~0.1 us per halving step; the
//   gather form 0.2 us per split (two cluster barriers, remote reads from
//   every split) plus the partial tile's width;
// - without split-K a dense call of full 256-token tiles with paired
//   channel blocks runs the CTA-pair form, whose deeper ring takes 0.22 us
//   per k tile instead of 0.29 (measured: one split then beats two on the
//   70B-like layers at M = 384..2048, and loses on the 4096-wide ones).
// Ties go to more splits.  W4A8_FORCE_SPLITS=<n> and W4A8_FORCE_TILE=<tokens>
// in the environment override the choice (tuning only).
Schedule choose_schedule(int M, int N, int K, int sms, bool w8, long active_m_tiles = 0,
                         int force_T = 0, int force_splits = 0) {
  Schedule s;
  s.T = force_T > 0 ? force_T : tile_tokens(M);
  static const int forced_tile = [] {  // tuning experiments only
    const char* e = getenv("W4A8_FORCE_TILE");
    return e ? atoi(e) : 0;
  }();
  if (force_T == 0 && (forced_tile == 16 || forced_tile == 32 || forced_tile == 64 ||
                       forced_tile == 128 || forced_tile == 256))
    s.T = forced_tile;
  s.n_tiles = (N + kTileN - 1) / kTileN;
  s.m_tiles = M > 0 ? (M + s.T - 1) / s.T : 0;
  const int kt = K / kTileK;
  // tiles that do work (grouped GEMMs launch more, which leave at once)
  const long tiles = (long)s.n_tiles * (active_m_tiles > 0 ? active_m_tiles : s.m_tiles);
  const double fill = s.T <= 64 ? 3.0 : s.T == 128 ? 6.0 : 7.4;
  const double t_cta = w8 ? (s.T == 16 ? 0.35 : s.T == 32 ? 0.40 : s.T == 64 ? 0.45 : 0.35)
                         : (s.T > 64 ? 0.29 : s.T == 16 ? 0.27 : 0.28);
  const double w_bytes = w8 ? (double)kTileN * kTileK : (double)kTileBytes;
  constexpr double kBytesPerUs = 6.0e6;  // sustained HBM read rate
  const bool push = s.T == 16 && M <= GemmCfg<16, 9, 4, 2, true>::kPushMaxM;
  static const int forced = [] {
    const char* e = getenv("W4A8_FORCE_SPLITS");
    return e ? atoi(e) : 0;
  }();
  const bool pair_ok = pair_enabled() && !w8 && active_m_tiles == 0 && s.T == 256 &&
                       s.n_tiles % 2 == 0 && M >= 256;
  double best = 1e300;
  for (int cand = 1; cand <= kMaxSplits && cand <= kt; ++cand) {
    const int per = (kt + cand - 1) / cand;
    const int eff = (kt + per - 1) / per;
    if (eff != cand) continue;  // same schedule as a smaller candidate
    const long slots = (long)sms * ctas_per_sm(s.T, per, w8);
    long per_wave = (eff & (eff - 1)) == 0 ? slots / eff : (long)(0.92 * slots / eff);
    if (per_wave < 1) per_wave = 1;
    const long waves = (tiles + per_wave - 1) / per_wave;
    const long resident = (tiles < per_wave ? tiles : per_wave) * eff;
    const double t_bw = resident * w_bytes / kBytesPerUs;
    const double t_own = (pair_ok && eff == 1) ? 0.22 : t_cta;
    const double t_tile = t_own > t_bw ? t_own : t_bw;
    const int lg = eff > 4 ? 3 : eff > 2 ? 2 : eff > 1 ? 1 : 0;
    const double tok = M < s.T ? M : s.T;
    // push: one async add per element into the leader, no barrier;
    // gather: two cluster barriers and remote reads across all splits
    const double red = eff == 1 ? 0.0 : push ? 0.1 * lg : 0.2 * eff + 0.05 * tok * lg / 8.0;
    double cost = waves * (fill + per * t_tile) + red;
    const int want = force_splits > 0 ? force_splits : forced;
    if (want > 0) cost = (eff == want) ? 0.0 : 1e6 + cost;
    if (cost <= best) {
      best = cost;
      s.splits = eff;
      s.kt_per = per;
    }
  }
  s.ctas = (int)((long)s.n_tiles * s.m_tiles * s.splits);
  return s;
}

// Grouped GEMM: token tiles are per group and the tile width comes from the
// bound on rows per group.  At most ceil(M_total / T) + groups - 1 token
// tiles hold rows (one partial tile per group), no more than M_total and no
// more than groups x ceil(max_rows / T); that many token-tile slots are
// launched (slots past the actual tiles leave at once) and the cost model
// counts them.  Schedule::m_tiles is the number of slots.
Schedule choose_grouped_schedule(int groups, int m_total, int max_rows, int N, int K, int sms) {
  Schedule s = choose_schedule(max_rows, N, K, sms, false);
  long slots = (m_total + s.T - 1) / s.T + groups - 1;
  if (slots > (long)groups * s.m_tiles) slots = (long)groups * s.m_tiles;
  if (slots > m_total) slots = m_total;
  s = choose_schedule(max_rows, N, K, sms, false, slots);
  s.m_tiles = (int)slots;
  s.ctas = (int)((long)s.n_tiles * s.m_tiles * s.splits);
  return s;
}

// ------------------------------------------------------------- launches
// Launch with optional programmatic dependent launch (PDL) and cluster size.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool pdl, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// Tensor maps of one launch: activations, and the INT8 weights (W8A8 only;
// a copy of the activation map stands in for the packed LQQ path).
struct Maps {
  CUtensorMap x, w;
};

template <int T, int SS, int AS, int DQG, int MINB, bool PUSH = false, bool W8 = false,
          int V = kVarDefault, bool PAIR = false, bool RTN = false, bool FUSED = false>
cudaError_t launch_gemm(const Maps& m, const GemmParams& p, int ctas, cudaStream_t st,
                        bool pdl) {
  using C = GemmCfg<T, SS, AS, DQG, PUSH, W8, PAIR, FUSED>;
  auto k = w4a8_gemm_kernel<T, SS, AS, DQG, MINB, PUSH, W8, V, PAIR, RTN, FUSED>;
  const cudaError_t ea = ensure_smem_attr<T, SS, AS, DQG, MINB, PUSH, W8, V, PAIR, RTN, FUSED>();
  if (ea != cudaSuccess) return ea;
  return launch_k(k, dim3(ctas), dim3(C::kThreads), C::kSmemBytes, st, pdl,
                  PAIR ? 2 : p.splits, m.x, m.w, p);
}

// The CTA-pair form of the 256-token tile (two CTAs share each token tile:
// each holds 128 channels and loads half of the tokens, so a stage is
// 16 KB of activations instead of 32 KB and the ring is 8 deep instead of
// 5): taken for dense calls without split-K whose channel blocks pair up
// and whose token tiles are full height.  (Grouped calls keep the
// single-CTA tile: on the Mixtral-like prefill the pair was 5% slower for
// the wide layer and 2% faster for the narrow one.)
// Bf16 tiles written by a TMA store from shared memory (dense calls without
// split-K).  W4A8_STORE_Y=0 in the environment turns it off (tuning only).
bool store_y_enabled() {
  static const bool enabled = [] {
    const char* v = getenv("W4A8_STORE_Y");
    return !(v && v[0] == '0');
  }();
  return enabled;
}

bool use_pair(const Schedule& s, const GemmParams& p, bool grouped) {
  return pair_enabled() && !grouped && s.T == 256 && s.splits == 1 && s.n_tiles % 2 == 0 &&
         p.M >= 256;
}

// ------------------------------------------------- persistent CTA pairs
// (gemm_pp.cuh): 192-token tiles, an 8-deep stage ring, 4 weight slots.
constexpr int kPpTW = 192, kPpSS = 8, kPpAS = 4;
using PpC = PpCfg<kPpTW, kPpSS, kPpAS>;

// Output tiles of the persistent form for a shape (channel-block pairs x
// 192-token tiles); 0 when N does not pad to whole pairs.
long pp_tiles(int M, int N) {
  const int n_tiles = (N + kTileN - 1) / kTileN;
  if (n_tiles % 2 != 0) return 0;
  return (long)(n_tiles / 2) * ((M + kPpTW - 1) / kPpTW);
}

// The persistent form for a dense call: bf16 output through a TMA store
// (N a multiple of 8, Y 16-byte aligned), or INT32 output.  Returns
// cudaErrorNotSupported (nothing launched) when the output does not qualify.
cudaError_t launch_pp(const int8_t* Xq, const float* s_x, const void* packed, int M, int N,
                      int K, uint16_t* Y, int32_t* acc, cudaStream_t st, bool pdl, int sms) {
  if (Y && (N % 8 != 0 || !aligned(Y, 16))) return cudaErrorNotSupported;
  const long tiles = pp_tiles(M, N);
  if (tiles <= 0) return cudaErrorNotSupported;
  const int n_pad = round_up(N, kTileN);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  PpParams p;
  p.tiles = base + tiles_offset_bytes(n_pad);
  p.s_w = reinterpret_cast<const float*>(base + sw_offset_bytes());
  p.s_x = s_x;
  p.acc = Y ? nullptr : acc;
  p.hdr = reinterpret_cast<const PackedHeader*>(base);
  p.M = M;
  p.N = N;
  p.K = K;
  p.kt_total = K / kTileK;
  p.n_pairs = n_pad / kTileN / 2;
  p.m_tiles = (M + kPpTW - 1) / kPpTW;
  p.m_band = p.m_tiles < kRasterBand ? p.m_tiles : kRasterBand;
  p.wait_limit_ns = wait_budget();
  CUtensorMap mx, my;
  if (!make_act_map(&mx, Xq, M, K, kPpTW / 2)) return cudaErrorInvalidValue;
  my = mx;
  if (Y && !make_y_map(&my, Y, M, N, kPpTW)) return cudaErrorInvalidValue;
  auto k = w4a8_gemm_pp_kernel<kPpTW, kPpSS, kPpAS>;
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PpC::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  const long pairs = tiles < sms / 2 ? tiles : sms / 2;
  return launch_k(k, dim3((unsigned)(2 * pairs)), dim3(PpC::kThreads), PpC::kSmemBytes, st, pdl,
                  2, mx, my, p);
}

// Pair launch: the activation box is the CTA's half of the token tile.
cudaError_t launch_pair(const int8_t* Xq, int M, int K, Maps& m, GemmParams& p, int ctas,
                        cudaStream_t st, bool pdl) {
  p.tn = round_up(p.tn, 32);  // each CTA loads tn / 2 rows
  if (!make_act_map(&m.x, Xq, M, K, p.tn / 2)) return cudaErrorInvalidValue;
  return p.tn == 256
             ? launch_gemm<256, 8, 4, 2, 1, false, false, kVarDefault, true>(m, p, ctas, st, pdl)
             : launch_gemm<256, 8, 4, 2, 1, false, false, kVarDefault, true, true>(m, p, ctas, st,
                                                                                   pdl);
}

// Checks shared by both weight formats; fills the launch-independent part
// of the parameters.  Returns W4A8_OK or an error (nothing launched).
int check_common(const int8_t* Xq, const float* s_x, const void* w, int M, int N, int K,
                 uint16_t* Y, int32_t* acc, unsigned flags) {
  if (flags & ~(unsigned)(W4A8_FLAG_PDL | W4A8_FLAG_TENSOR_CORE)) return W4A8_ERR_INVALID_ARG;
  if (M < 0 || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return W4A8_OK;
  if (!Xq || !w || (!Y && !acc) || (Y && !s_x)) return W4A8_ERR_INVALID_ARG;
  if (!aligned(Xq, 16) || !aligned(w, 16) || (Y && !aligned(Y, 2)) ||
      (acc && !aligned(acc, 4)) || (s_x && !aligned(s_x, 4)))
    return W4A8_ERR_MISALIGNED;
  return W4A8_OK;
}

// Activation box of a single-CTA tile: only rows that exist are fetched when
// M < tn (the MMA still reads tn rows, but rows past M only feed accumulator
// columns that are never stored).  The kernel expects exactly these bytes.
int box_rows(const GemmParams& p) { return p.M < p.tn ? p.M : p.tn; }

GemmParams make_params(const Schedule& s, const float* s_x, int M, int N, int K, uint16_t* Y,
                       int32_t* acc) {
  GemmParams p;
  p.tiles = nullptr;
  p.s_w = nullptr;
  p.s_x = s_x;
  p.Y = Y;
  p.acc = Y ? nullptr : acc;
  p.M = M;
  p.N = N;
  p.K = K;
  p.n_pad = round_up(N, kTileN);
  p.kt_total = K / kTileK;
  p.splits = s.splits;
  p.kt_per_split = s.kt_per;
  p.n_tiles = s.n_tiles;
  p.m_tiles = s.m_tiles;
  p.wait_limit_ns = wait_budget();
  p.hdr = nullptr;
  p.offsets = nullptr;
  p.group_bytes = 0;
  p.m_total = M;
  p.groups = 0;
  // Bands of up to 8 token tiles: a wave of 148 CTAs then spans about 18
  // channel blocks x 8 token tiles, whose weights and activations stay in
  // L2 while the wave reuses them.  Weights read by one token tile only are
  // streamed with an evict-first hint.
  p.m_band = s.m_tiles < kRasterBand ? s.m_tiles : kRasterBand;
  p.mode = s.m_tiles == 1 ? kModeStreamW : 0;
  // The 256-token configurations size the tile to the rows: the token tiles
  // share M evenly, rounded up to the MMA's granularity of 16.
  p.tn = s.T;
  if (s.T == 256 && s.m_tiles > 0) p.tn = round_up((M + s.m_tiles - 1) / s.m_tiles, 16);
  return p;
}

// ------------------------------------------------ CUDA-core decode form
// (gemv.cuh): R = 16 channels per CTA, P = 8 pieces per thread, so a CTA
// covers at most 32 k tiles (K = 4096); longer rows split K across a cluster.
constexpr int kGemvR = 16, kGemvP = 8, kGemvMinB = 2;
using GemvC = GemvCfg<kGemvR, kGemvP>;
// the warp-MMA form covers the same CTA slice (16 channels x 32 k tiles)
using GemvMmaC = GemvMmaCfg<GemvC::kKR>;
static_assert(GemvMmaC::kR == kGemvR, "one tensor-map box for both decode forms");

struct GemvSchedule {
  int splits = 1, kt_per = 1, ctas = 0;
};

// Whether a decode form applies to a shape: up to 16 tokens for the
// warp-MMA form, 8 for the dp4a one (fused: one split only, the CTA then
// holds whole rows of X for the per-token absmax).
bool gemv_schedule(int M, int N, int K, bool fused, GemvSchedule* out, bool mma = true) {
  const int max_m = mma ? kGemvMmaMaxM : kGemvMaxM;
  if (M < 1 || M > max_m || N < 1 || K < kTileK || K % kTileK != 0 || K > 65536)
    return false;
  const int kt = K / kTileK;
  const int splits = (kt + GemvC::kKR - 1) / GemvC::kKR;
  if (splits > kGemvMaxSplits || (fused && splits > 1)) return false;
  GemvSchedule s;
  s.splits = splits;
  s.kt_per = (kt + splits - 1) / splits;
  s.ctas = round_up(N, kTileN) / kGemvR * splits;
  if (out) *out = s;
  return true;
}

// W4A8_GEMV=0 in the environment never takes the CUDA-core form, =1 takes
// it wherever it applies (tuning experiments only).
int gemv_env() {
  static const int v = [] {
    const char* e = getenv("W4A8_GEMV");
    return e ? (e[0] == '0' ? 0 : 1) : -1;
  }();
  return v;
}

// Default choice between the decode form and the tcgen05 kernel: the decode
// form when all its CTAs are resident at once (two per SM), so that every
// CTA fetches and dequantizes its weights before the preceding kernel
// finishes.  Measured on B200 (graphs of back-to-back calls with
// programmatic dependent launch): N = K = 4096, M = 1..8: 4.6-4.8 us
// against 5.0-5.7 us, and 6.0-6.7 us against 6.3-8.5 us per quantize +
// GEMM pair; with several waves of CTAs (7B- and 70B-like layers) each
// wave waits for its weights and the tcgen05 kernel is 1.5-2.5x faster.
bool prefer_gemv(int M, int N, int K) {
  GemvSchedule s;
  if (!gemv_schedule(M, N, K, false, &s)) return false;
  const int env = gemv_env();
  if (env >= 0) return env == 1;
  int dev = 0;
  const int sms = cudaGetDevice(&dev) == cudaSuccess ? num_sms(dev) : 148;
  return s.ctas <= kGemvMinB * sms;
}

// Tensor maps over the packed tiles for one CTA's box: the codes as a 4-D
// array [channel block][k tile][chunk][128 rows x 16 bytes] (box: R rows x 4
// chunks x KR k tiles), the (s_u8, a) pairs as a 3-D array [channel block]
// [k tile][128 rows x 4 bytes] starting 8192 bytes into each tile.  Boxes
// past the last k tile are zero-filled; those k tiles are never used.
bool make_gemv_maps(const uint8_t* tiles, int n_pad, int kt_total, CUtensorMap* codes,
                    CUtensorMap* prm) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t nblk = (cuuint64_t)(n_pad / kTileN);
  const cuuint64_t tile = kTileBytes, block = (cuuint64_t)kt_total * kTileBytes;
  {
    cuuint64_t dims[4] = {(cuuint64_t)kTileN * 16, 4, (cuuint64_t)kt_total, nblk};
    cuuint64_t strides[3] = {(cuuint64_t)kTileN * 16, tile, block};
    cuuint32_t box[4] = {(cuuint32_t)(kGemvR * 16), 4, (cuuint32_t)GemvC::kKR, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (fn(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(tiles), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)kTileN * 4, (cuuint64_t)kt_total, nblk};
    cuuint64_t strides[2] = {tile, block};
    cuuint32_t box[3] = {(cuuint32_t)(kGemvR * 4), (cuuint32_t)GemvC::kKR, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(prm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(tiles) + kCodeBytes,
           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// MMA: the warp-MMA kernel (the library's decode form; NG groups of 8
// tokens), else the dp4a one (ablation).
template <bool MMA, int NG, bool FUSED>
cudaError_t launch_gemv(const GemvParams& p, const GemvSchedule& s, const uint8_t* tiles,
                        int n_pad, cudaStream_t st, bool pdl) {
  auto k = MMA ? w4a8_gemv_mma_kernel<GemvC::kKR, NG, kGemvMinB, FUSED>
               : w4a8_gemv_kernel<kGemvR, kGemvP, kGemvMinB, FUSED>;
  const int smem_max =
      MMA ? GemvMmaC::smem_bytes(8 * NG) : GemvC::smem_bytes(kGemvMaxM);
  const int smem = MMA ? GemvMmaC::smem_bytes(p.M) : GemvC::smem_bytes(p.M);
  static std::atomic<bool> attr_set[kMaxDevices];
  const int dev = current_device();
  if (dev >= 0 && dev < kMaxDevices && !attr_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_relaxed);
  }
  CUtensorMap codes, prm;
  if (!make_gemv_maps(tiles, n_pad, p.kt_total, &codes, &prm)) return cudaErrorInvalidValue;
  return launch_k(k, dim3(s.ctas), dim3(kGemvThreads), smem, st, pdl, s.splits, codes, prm, p);
}

// The decode form of a dense call (X fp32 when fused, else Xq / s_x); mma
// picks the warp-MMA kernel, else the dp4a one.
int gemm_gemv(const int8_t* Xq, const float* X, const float* s_x, const void* packed, int M,
              int N, int K, uint16_t* Y, int32_t* acc, bool pdl, void* stream, bool mma = true) {
  GemvSchedule s;
  const bool fused = X != nullptr;
  if (!gemv_schedule(M, N, K, fused, &s, mma)) return W4A8_ERR_UNSUPPORTED_SHAPE;
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  const int n_pad = round_up(N, kTileN);
  GemvParams p;
  p.Xq = Xq;
  p.X = X;
  p.s_x = s_x;
  p.s_w = reinterpret_cast<const float*>(base + sw_offset_bytes());
  p.hdr = reinterpret_cast<const PackedHeader*>(base);
  p.Y = Y;
  p.acc = Y ? nullptr : acc;
  p.M = M;
  p.N = N;
  p.K = K;
  p.kt_total = K / kTileK;
  p.splits = s.splits;
  p.kt_per = s.kt_per;
  p.wait_limit_ns = wait_budget();
  const uint8_t* tiles = base + tiles_offset_bytes(n_pad);
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  if (!mma)
    e = fused ? launch_gemv<false, 1, true>(p, s, tiles, n_pad, st, pdl)
              : launch_gemv<false, 1, false>(p, s, tiles, n_pad, st, pdl);
  else if (M <= 8)
    e = fused ? launch_gemv<true, 1, true>(p, s, tiles, n_pad, st, pdl)
              : launch_gemv<true, 1, false>(p, s, tiles, n_pad, st, pdl);
  else
    e = fused ? launch_gemv<true, 2, true>(p, s, tiles, n_pad, st, pdl)
              : launch_gemv<true, 2, false>(p, s, tiles, n_pad, st, pdl);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// Grouped (mixture-of-experts) form of a call; groups == 0 for a dense GEMM.
struct Groups {
  int groups = 0;
  const int* offsets = nullptr;
  int m_total = 0;
};

// W4A8 GEMM, dense (M rows) or grouped (g.m_total rows in g.groups groups of
// at most M rows each).
// Kernel paths of a dense call: the library's choice, or one forced (the
// tensor-core kernel, or the CUDA-core decode form).
enum class Path { kAuto, kTensor, kWarpMma, kDp4a, kPersist };

int gemm_common(const int8_t* Xq, const float* s_x, const void* packed, int M, int N,
                int K, uint16_t* Y, int32_t* acc, unsigned flags, void* stream,
                const Groups& g = Groups(), Path path = Path::kAuto) {
  const int rc = check_common(Xq, s_x, packed, M, N, K, Y, acc, flags);
  if (rc != W4A8_OK || M == 0) return rc;
  const bool pdl = (flags & W4A8_FLAG_PDL) != 0;
  if (flags & W4A8_FLAG_TENSOR_CORE) path = Path::kTensor;
  if (g.groups == 0 && path == Path::kDp4a)
    return gemm_gemv(Xq, nullptr, s_x, packed, M, N, K, Y, acc, pdl, stream, false);
  if (g.groups == 0 && path == Path::kPersist) {  // forced (tests, ablation): any M
    const int d = current_device();
    if (d < 0) return W4A8_ERR_CUDA;
    const cudaError_t e =
        launch_pp(Xq, s_x, packed, M, N, K, Y, acc, as_stream(stream), pdl, num_sms(d));
    return e == cudaSuccess ? W4A8_OK
                            : e == cudaErrorNotSupported ? W4A8_ERR_UNSUPPORTED_SHAPE
                                                         : W4A8_ERR_CUDA;
  }
  if (g.groups == 0 &&
      (path == Path::kWarpMma || (path == Path::kAuto && prefer_gemv(M, N, K))))
    return gemm_gemv(Xq, nullptr, s_x, packed, M, N, K, Y, acc, pdl, stream, true);
  const int dev = current_device();
  if (dev < 0) return W4A8_ERR_CUDA;
  const Schedule s = g.groups > 0 ? choose_grouped_schedule(g.groups, g.m_total, M, N, K,
                                                            num_sms(dev))
                                  : choose_schedule(M, N, K, num_sms(dev), false);
  GemmParams p = make_params(s, s_x, M, N, K, Y, acc);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  p.tiles = base + tiles_offset_bytes(p.n_pad);
  p.s_w = reinterpret_cast<const float*>(base + sw_offset_bytes());
  p.hdr = reinterpret_cast<const PackedHeader*>(base);
  const int x_rows = g.groups > 0 ? g.m_total : M;  // rows of Xq / Y
  if (g.groups > 0) {
    p.offsets = g.offsets;
    p.group_bytes = (size_t)packed_bytes(N, K);
    p.m_total = g.m_total;
    p.groups = g.groups;
    p.m_band = 1;
    // groups of up to 256 rows take one tile of their bound's width
    if (s.T == 256) p.tn = round_up(M < 256 ? M : 256, 16);
    p.mode = M <= p.tn ? kModeStreamW : 0;  // one token tile per group
  }

  const bool pair = s.T == 256 && use_pair(s, p, g.groups > 0);
  if (pair) p.tn = round_up(p.tn, 32);  // each CTA of a pair loads tn / 2 rows

  Maps m;
  // the box holds min(T, M) rows: every valid row of a tile (grouped: M
  // bounds each group's rows), and exactly the bytes the kernel expects
  if (!make_act_map(&m.x, Xq, x_rows, K, box_rows(p))) return W4A8_ERR_CUDA;
  m.w = m.x;
  // Dense calls without split-K write their bf16 tile with one TMA store
  // (the second tensor map); the box is the CTA's tile rows.
  if (g.groups == 0 && Y && s.splits == 1 && N % 8 == 0 && aligned(Y, 16) && store_y_enabled() &&
      make_y_map(&m.w, Y, M, N, pair ? p.tn : box_rows(p)))
    p.mode |= kModeStoreY;
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  switch (s.T) {
    // (tokens, smem stages, TMEM A slots, dequant groups, CTAs per SM[, push])
    case 16: {
      // Short k ranges (<= 6 tiles per CTA) use a light ring that fits three
      // CTAs per SM, so a following launch's CTAs find room early and start
      // fetching weights under programmatic dependent launch; long ones keep
      // the deep ring.  Split decode with at most 8 tokens pushes partials
      // (8 KB receive buffer).
      const bool push = s.splits > 1 && M <= GemmCfg<16, 9, 4, 2, true>::kPushMaxM;
      if (ctas_per_sm(16, s.kt_per, false) == 3)
        e = push ? launch_gemm<16, 6, 3, 2, 3, true>(m, p, s.ctas, st, pdl)
                 : launch_gemm<16, 6, 3, 2, 3>(m, p, s.ctas, st, pdl);
      else
        e = push ? launch_gemm<16, 9, 4, 2, 2, true>(m, p, s.ctas, st, pdl)
                 : launch_gemm<16, 10, 4, 2, 2>(m, p, s.ctas, st, pdl);
      break;
    }
    // (the 64-token tile fills its 256 TMEM columns with A slots: more weight
    // tiles dequantized before the activations land, 4-6% faster at M = 64 on
    // short and long k ranges.  The 16- and 32-token rings keep 4: deeper
    // measured 2-8% slower on the long k ranges of the 70B-like decode layers)
    case 32: e = launch_gemm<32, 8, 4, 2, 2>(m, p, s.ctas, st, pdl); break;
    case 64: e = launch_gemm<64, 6, 6, 2, 2>(m, p, s.ctas, st, pdl); break;
    case 128: e = launch_gemm<128, 4, 4, 2, 2>(m, p, s.ctas, st, pdl); break;  // tuning only
    default:
      if (pair)
        e = launch_pair(Xq, x_rows, K, m, p, s.ctas, st, pdl);
      else if (p.tn == 256)
        e = launch_gemm<256, 5, 4, 2, 1>(m, p, s.ctas, st, pdl);
      else
        e = launch_gemm<256, 5, 4, 2, 1, false, false, kVarDefault, false, true>(m, p, s.ctas,
                                                                                st, pdl);
      break;
  }
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// The W8A8 comparison GEMM: the same kernel with plain INT8 weights read by
// the MMA from shared memory (no dequantization warps: one group of four
// epilogue warps).
int gemm_w8_common(const int8_t* Xq, const float* s_x, const int8_t* Wq, const float* s_w,
                   int M, int N, int K, uint16_t* Y, int32_t* acc, unsigned flags,
                   void* stream) {
  if (flags & ~(unsigned)W4A8_FLAG_PDL) return W4A8_ERR_INVALID_ARG;  // (one kernel only)
  const int rc = check_common(Xq, s_x, Wq, M, N, K, Y, acc, flags);
  if (rc != W4A8_OK || M == 0) return rc;
  if (Y && !s_w) return W4A8_ERR_INVALID_ARG;
  if (s_w && !aligned(s_w, 4)) return W4A8_ERR_MISALIGNED;
  const bool pdl = (flags & W4A8_FLAG_PDL) != 0;
  const int dev = current_device();
  if (dev < 0) return W4A8_ERR_CUDA;
  const Schedule s = choose_schedule(M, N, K, num_sms(dev), true);
  GemmParams p = make_params(s, s_x, M, N, K, Y, acc);
  p.s_w = s_w;
  p.tn = s.T;  // the W8A8 kernel keeps whole tiles

  Maps m;
  if (!make_act_map(&m.x, Xq, M, K, box_rows(p))) return W4A8_ERR_CUDA;
  if (!make_w8_map(&m.w, Wq, N, K)) return W4A8_ERR_CUDA;
  cudaStream_t st = as_stream(stream);
  cudaError_t e;
  switch (s.T) {
    // (tokens, smem stages, -, epilogue groups, CTAs per SM, push, W8)
    case 16: {
      const bool push = s.splits > 1 && M <= GemmCfg<16, 5, 1, 1, true, true>::kPushMaxM;
      e = push ? launch_gemm<16, 5, 1, 1, 2, true, true>(m, p, s.ctas, st, pdl)
               : launch_gemm<16, 6, 1, 1, 2, false, true>(m, p, s.ctas, st, pdl);
      break;
    }
    case 32: e = launch_gemm<32, 5, 1, 1, 2, false, true>(m, p, s.ctas, st, pdl); break;
    case 64: e = launch_gemm<64, 4, 1, 1, 2, false, true>(m, p, s.ctas, st, pdl); break;
    case 128: e = launch_gemm<128, 3, 1, 1, 2, false, true>(m, p, s.ctas, st, pdl); break;
    default: e = launch_gemm<256, 4, 1, 1, 1, false, true>(m, p, s.ctas, st, pdl); break;
  }
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// Ablation study: the same product through kernel variants that each change
// one design decision against a fixed baseline configuration (16-token tile
// with the deep ring for M <= 16, else the 256-token tile; gather split-K
// reduction; the library's schedule).
int gemm_variant(int variant, const int8_t* Xq, const float* s_x, const void* packed, int M,
                 int N, int K, uint16_t* Y, int32_t* acc, unsigned flags, void* stream) {
  if (variant < W4A8_VARIANT_DEFAULT || variant > W4A8_VARIANT_PERSISTENT)
    return W4A8_ERR_INVALID_ARG;
  if (variant == W4A8_VARIANT_PERSISTENT)
    return gemm_common(Xq, s_x, packed, M, N, K, Y, acc, flags, stream, Groups(),
                       Path::kPersist);
  if (variant == W4A8_VARIANT_DEFAULT)
    return gemm_common(Xq, s_x, packed, M, N, K, Y, acc, flags, stream);
  if (variant == W4A8_VARIANT_TENSOR_CORE)
    return gemm_common(Xq, s_x, packed, M, N, K, Y, acc, flags, stream, Groups(), Path::kTensor);
  if (variant == W4A8_VARIANT_DP4A || variant == W4A8_VARIANT_WARP_MMA) {
    const int rc0 = check_common(Xq, s_x, packed, M, N, K, Y, acc, flags);
    if (rc0 != W4A8_OK || M == 0) return rc0;
    if (!gemv_schedule(M, N, K, false, nullptr, variant == W4A8_VARIANT_WARP_MMA))
      return W4A8_ERR_UNSUPPORTED_SHAPE;
    return gemm_common(Xq, s_x, packed, M, N, K, Y, acc, flags, stream, Groups(),
                       variant == W4A8_VARIANT_DP4A ? Path::kDp4a : Path::kWarpMma);
  }
  const int rc = check_common(Xq, s_x, packed, M, N, K, Y, acc, flags);
  if (rc != W4A8_OK || M == 0) return rc;
  const bool pdl = (flags & W4A8_FLAG_PDL) != 0;
  const int dev = current_device();
  if (dev < 0) return W4A8_ERR_CUDA;
  const int T = M <= 16 ? 16 : 256;
  const bool pair = variant == W4A8_VARIANT_CTA_PAIR;
  if (pair && (T != 256 || ((N + kTileN - 1) / kTileN) % 2 != 0 || M < 256))
    return W4A8_ERR_UNSUPPORTED_SHAPE;
  const Schedule s = choose_schedule(M, N, K, num_sms(dev), false, 0, T, pair ? 1 : 0);
  GemmParams p = make_params(s, s_x, M, N, K, Y, acc);
  if (!pair) {
    p.tn = s.T;  // the ablation variants keep whole tiles
    }
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  p.tiles = base + tiles_offset_bytes(p.n_pad);
  p.s_w = reinterpret_cast<const float*>(base + sw_offset_bytes());
  p.hdr = reinterpret_cast<const PackedHeader*>(base);
  Maps m;
  if (!make_act_map(&m.x, Xq, M, K, box_rows(p))) return W4A8_ERR_CUDA;
  m.w = m.x;
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaErrorInvalidValue;
  // (tokens, smem stages, TMEM A slots, dequant groups, CTAs per SM, push, W8, variant)
  if (T == 16) {
    switch (variant) {
      case W4A8_VARIANT_BASELINE: e = launch_gemm<16, 10, 4, 2, 2>(m, p, s.ctas, st, pdl); break;
      case W4A8_VARIANT_NAIVE_DEQUANT:
        e = launch_gemm<16, 10, 4, 2, 2, false, false, kVarNaiveDequant>(m, p, s.ctas, st, pdl);
        break;
      case W4A8_VARIANT_SERIAL: e = launch_gemm<16, 10, 1, 1, 2>(m, p, s.ctas, st, pdl); break;
      case W4A8_VARIANT_ONE_GROUP: e = launch_gemm<16, 10, 4, 1, 2>(m, p, s.ctas, st, pdl); break;
      default:
        e = launch_gemm<16, 10, 4, 1, 2, false, false, kVarGroupIssuesMma>(m, p, s.ctas, st, pdl);
        break;
    }
  } else if (pair) {
    e = launch_pair(Xq, M, K, m, p, s.ctas, st, pdl);
  } else {
    switch (variant) {
      case W4A8_VARIANT_BASELINE: e = launch_gemm<256, 5, 4, 2, 1>(m, p, s.ctas, st, pdl); break;
      case W4A8_VARIANT_NAIVE_DEQUANT:
        e = launch_gemm<256, 5, 4, 2, 1, false, false, kVarNaiveDequant>(m, p, s.ctas, st, pdl);
        break;
      case W4A8_VARIANT_SERIAL: e = launch_gemm<256, 5, 1, 1, 1>(m, p, s.ctas, st, pdl); break;
      case W4A8_VARIANT_ONE_GROUP: e = launch_gemm<256, 5, 4, 1, 1>(m, p, s.ctas, st, pdl); break;
      default:
        e = launch_gemm<256, 5, 4, 1, 1, false, false, kVarGroupIssuesMma>(m, p, s.ctas, st, pdl);
        break;
    }
  }
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

// Whether the fused form (activation quantization inside the GEMM) applies:
// the 16-token light ring with every k tile of a CTA resident, and split-K
// only with the push reduction.
bool fused_schedule(int M, int N, int K, int sms, Schedule* out) {
  if (M < 1 || M > 16 || N < 1 || K % kTileK != 0 || K > 65536) return false;
  const Schedule s = choose_schedule(M, N, K, sms, false);
  if (s.T != 16 || ctas_per_sm(16, s.kt_per, false) != 3 || s.kt_per > 6) return false;
  if (s.splits > 1 && M > GemmCfg<16, 6, 3, 2, true>::kPushMaxM) return false;
  // the CTA's slice of X (M rows x kt_per k tiles) sits in the two quantizing
  // warps' registers
  using F = GemmCfg<16, 6, 3, 2, true, false, false, true>;
  if (M * s.kt_per * (kTileK / 4) > 64 * F::kFusedV) return false;
  if (out) *out = s;
  return true;
}

int gemm_fused(const float* X, const void* packed, int M, int N, int K, uint16_t* Y,
               unsigned flags, void* stream) {
  if (flags & ~(unsigned)(W4A8_FLAG_PDL | W4A8_FLAG_TENSOR_CORE)) return W4A8_ERR_INVALID_ARG;
  if (M < 0 || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return W4A8_OK;
  if (!X || !packed || !Y) return W4A8_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(packed, 16) || !aligned(Y, 2)) return W4A8_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return W4A8_ERR_CUDA;
  // a few tokens with whole rows per CTA: the CUDA-core form quantizes in
  // each CTA; otherwise the tensor-core form with its quantizing warps
  if (!(flags & W4A8_FLAG_TENSOR_CORE) && gemv_schedule(M, N, K, true, nullptr) &&
      gemv_env() != 0)
    return gemm_gemv(nullptr, X, nullptr, packed, M, N, K, Y, nullptr,
                     (flags & W4A8_FLAG_PDL) != 0, stream);
  Schedule s;
  if (!fused_schedule(M, N, K, num_sms(dev), &s)) return W4A8_ERR_UNSUPPORTED_SHAPE;
  GemmParams p = make_params(s, reinterpret_cast<const float*>(X), M, N, K, Y, nullptr);
  const uint8_t* base = static_cast<const uint8_t*>(packed);
  p.tiles = base + tiles_offset_bytes(p.n_pad);
  p.s_w = reinterpret_cast<const float*>(base + sw_offset_bytes());
  p.hdr = reinterpret_cast<const PackedHeader*>(base);
  Maps m = {};  // no activation tensor map: the kernel reads X itself
  const bool push = s.splits > 1;
  const bool pdl = (flags & W4A8_FLAG_PDL) != 0;
  cudaStream_t st = as_stream(stream);
  const cudaError_t e =
      push ? launch_gemm<16, 6, 3, 2, 3, true, false, kVarDefault, false, false, true>(
                 m, p, s.ctas, st, pdl)
           : launch_gemm<16, 6, 3, 2, 3, false, false, kVarDefault, false, false, true>(
                 m, p, s.ctas, st, pdl);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

__global__ void timeout_probe_kernel(unsigned long long limit_ns) {
  __shared__ alignas(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  // nothing ever arrives on this barrier: the bounded wait must give up
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, nullptr, limit_ns);
}

}  // namespace
}  // namespace w4a8

using namespace w4a8;

extern "C" {

const char* w4a8_status_string(int status) {
  switch (status) {
    case W4A8_OK: return "W4A8_OK";
    case W4A8_ERR_INVALID_ARG: return "W4A8_ERR_INVALID_ARG";
    case W4A8_ERR_UNSUPPORTED_SHAPE: return "W4A8_ERR_UNSUPPORTED_SHAPE";
    case W4A8_ERR_MISALIGNED: return "W4A8_ERR_MISALIGNED";
    case W4A8_ERR_CUDA: return "W4A8_ERR_CUDA";
    case W4A8_ERR_TIMEOUT: return "W4A8_ERR_TIMEOUT";
    case W4A8_ERR_BAD_PACKED: return "W4A8_ERR_BAD_PACKED";
    case W4A8_ERR_BAD_OFFSETS: return "W4A8_ERR_BAD_OFFSETS";
    default: return "W4A8_ERR_UNKNOWN";
  }
}

int w4a8_version(void) { return 1; }

size_t w4a8_packed_weight_bytes(int N, int K, int group) {
  if (N < 1 || K < 1 || K % kTileK != 0 || K > 65536 || (group != 64 && group != 128))
    return 0;
  return (size_t)packed_bytes(N, K);
}

int w4a8_quantize_weights(const float* W, int N, int K, int group, void* packed,
                          void* stream) {
  if (!W || !packed || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (group != 64 && group != 128) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(W, 16) || !aligned(packed, 16)) return W4A8_ERR_MISALIGNED;
  const int dev = current_device();
  if (dev < 0) return W4A8_ERR_CUDA;
  const int n_pad = round_up(N, kTileN);
  cudaStream_t st = as_stream(stream);
  uint8_t* out = static_cast<uint8_t*>(packed);
  weight_scale_kernel<<<(n_pad + 7) / 8, 256, 0, st>>>(W, N, K, group, n_pad, out);
  if (cudaGetLastError() != cudaSuccess) return W4A8_ERR_CUDA;
  static std::atomic<bool> attr_set[kMaxDevices];
  if (dev < kMaxDevices && !attr_set[dev].load()) {
    if (cudaFuncSetAttribute(weight_pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kPackSmemBytes) != cudaSuccess)
      return W4A8_ERR_CUDA;
    attr_set[dev].store(true);
  }
  dim3 grid(K / kTileK, n_pad / kTileN);
  weight_pack_kernel<<<grid, 128, kPackSmemBytes, st>>>(W, N, K, group, n_pad, out);
  return cudaGetLastError() == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

int w4a8_unpack_weights(const void* packed, int N, int K, uint8_t* codes, uint8_t* s_u8,
                        uint8_t* a, float* s_w, void* stream) {
  if (!packed || !codes || !s_u8 || !a || !s_w || N < 1 || K < 1)
    return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(packed, 16) || !aligned(s_w, 4)) return W4A8_ERR_MISALIGNED;
  const int n_pad = round_up(N, kTileN);
  dim3 grid(K / kTileK, n_pad / kTileN);
  weight_unpack_kernel<<<grid, 128, 0, as_stream(stream)>>>(
      static_cast<const uint8_t*>(packed), N, K, n_pad, codes, s_u8, a, s_w);
  return cudaGetLastError() == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

int w4a8_quantize_act(const float* X, int M, int K, int8_t* Xq, float* s_x, void* stream) {
  return w4a8_quantize_act_ex(X, M, K, Xq, s_x, 0u, stream);
}

int w4a8_quantize_act_ex(const float* X, int M, int K, int8_t* Xq, float* s_x, unsigned flags,
                         void* stream) {
  if (flags & ~(unsigned)W4A8_FLAG_PDL) return W4A8_ERR_INVALID_ARG;
  if (M < 0 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % 16 != 0) return W4A8_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return W4A8_OK;
  if (!X || !Xq || !s_x) return W4A8_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(Xq, 16) || !aligned(s_x, 4)) return W4A8_ERR_MISALIGNED;
  cudaError_t e = launch_k(act_quant_kernel, dim3(M), dim3(kActThreads), 0, as_stream(stream),
                           (flags & W4A8_FLAG_PDL) != 0, 1, X, M, K, Xq, s_x);
  return e == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

int w4a8_gemm(const int8_t* Xq, const float* s_x, const void* packed, int M, int N, int K,
              uint16_t* Y, void* stream) {
  return gemm_common(Xq, s_x, packed, M, N, K, Y, nullptr, 0u, stream);
}

int w4a8_gemm_ex(const int8_t* Xq, const float* s_x, const void* packed, int M, int N, int K,
                 uint16_t* Y, unsigned flags, void* stream) {
  return gemm_common(Xq, s_x, packed, M, N, K, Y, nullptr, flags, stream);
}

int w4a8_gemm_i32(const int8_t* Xq, const void* packed, int M, int N, int K, int32_t* acc,
                  void* stream) {
  return gemm_common(Xq, nullptr, packed, M, N, K, nullptr, acc, 0u, stream);
}

int w4a8_gemm_schedule(int M, int N, int K, int* tile_tokens, int* splits, int* ctas) {
  if (M < 0 || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  GemvSchedule gs;
  if (M > 0 && prefer_gemv(M, N, K) && gemv_schedule(M, N, K, false, &gs)) {
    if (tile_tokens) *tile_tokens = M;
    if (splits) *splits = gs.splits;
    if (ctas) *ctas = gs.ctas;
    return W4A8_OK;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const Schedule s = choose_schedule(M, N, K, dev < 0 ? 148 : num_sms(dev), false);
  if (tile_tokens) *tile_tokens = s.T;
  if (splits) *splits = s.splits;
  if (ctas) *ctas = s.ctas;
  return W4A8_OK;
}

int w4a8_gemm_kernel_kind(int M, int N, int K) {
  if (M < 0 || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  return M > 0 && prefer_gemv(M, N, K) ? W4A8_KERNEL_WARP_MMA : W4A8_KERNEL_TENSOR_CORE;
}

int w4a8_grouped_gemm(const int8_t* Xq, const float* s_x, const void* packed, int groups,
                      const int* offsets, int M_total, int max_rows, int N, int K, uint16_t* Y,
                      unsigned flags, void* stream) {
  if (groups < 1 || M_total < 0 || max_rows < 0 || max_rows > M_total) return W4A8_ERR_INVALID_ARG;
  if (M_total == 0) return (flags & ~(unsigned)W4A8_FLAG_PDL) ? W4A8_ERR_INVALID_ARG : W4A8_OK;
  if (max_rows == 0 || !offsets || !Y) return W4A8_ERR_INVALID_ARG;
  if (!aligned(offsets, 4)) return W4A8_ERR_MISALIGNED;
  Groups g;
  g.groups = groups;
  g.offsets = offsets;
  g.m_total = M_total;
  return gemm_common(Xq, s_x, packed, max_rows, N, K, Y, nullptr, flags, stream, g);
}

int w4a8_grouped_gemm_i32(const int8_t* Xq, const void* packed, int groups, const int* offsets,
                          int M_total, int max_rows, int N, int K, int32_t* acc, void* stream) {
  if (groups < 1 || M_total < 0 || max_rows < 0 || max_rows > M_total) return W4A8_ERR_INVALID_ARG;
  if (M_total == 0) return W4A8_OK;
  if (max_rows == 0 || !offsets || !acc) return W4A8_ERR_INVALID_ARG;
  if (!aligned(offsets, 4)) return W4A8_ERR_MISALIGNED;
  Groups g;
  g.groups = groups;
  g.offsets = offsets;
  g.m_total = M_total;
  return gemm_common(Xq, nullptr, packed, max_rows, N, K, nullptr, acc, 0u, stream, g);
}

int w4a8_grouped_gemm_schedule(int groups, int M_total, int max_rows, int N, int K,
                               int* tile_tokens, int* splits, int* ctas) {
  if (groups < 1 || M_total < 1 || max_rows < 1 || max_rows > M_total || N < 1 || K < 1)
    return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const Schedule s =
      choose_grouped_schedule(groups, M_total, max_rows, N, K, dev < 0 ? 148 : num_sms(dev));
  if (tile_tokens) *tile_tokens = s.T;
  if (splits) *splits = s.splits;
  if (ctas) *ctas = s.ctas;
  return W4A8_OK;
}

int w4a8_gemm_variant(int variant, const int8_t* Xq, const float* s_x, const void* packed, int M,
                      int N, int K, uint16_t* Y, int32_t* acc, unsigned flags, void* stream) {
  if (Y && acc) return W4A8_ERR_INVALID_ARG;
  return gemm_variant(variant, Xq, s_x, packed, M, N, K, Y, acc, flags, stream);
}

int w4a8_gemm_fused(const float* X, const void* packed, int M, int N, int K, uint16_t* Y,
                    unsigned flags, void* stream) {
  return gemm_fused(X, packed, M, N, K, Y, flags, stream);
}

int w4a8_gemm_fused_supported(int M, int N, int K) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  return (gemv_schedule(M, N, K, true, nullptr) && gemv_env() != 0) ||
                 fused_schedule(M, N, K, dev < 0 ? 148 : num_sms(dev), nullptr)
             ? 1
             : 0;
}

int w8a8_quantize_weights(const float* W, int N, int K, int8_t* Wq, float* s_w, void* stream) {
  // per-channel symmetric INT8: the per-row rule of the activation quantizer
  if (N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  return w4a8_quantize_act_ex(W, N, K, Wq, s_w, 0u, stream);
}

int w8a8_gemm(const int8_t* Xq, const float* s_x, const int8_t* Wq, const float* s_w, int M,
              int N, int K, uint16_t* Y, unsigned flags, void* stream) {
  return gemm_w8_common(Xq, s_x, Wq, s_w, M, N, K, Y, nullptr, flags, stream);
}

int w8a8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K, int32_t* acc,
                  void* stream) {
  return gemm_w8_common(Xq, nullptr, Wq, nullptr, M, N, K, nullptr, acc, 0u, stream);
}

int w8a8_gemm_schedule(int M, int N, int K, int* tile_tokens, int* splits, int* ctas) {
  if (M < 0 || N < 1 || K < 1) return W4A8_ERR_INVALID_ARG;
  if (K % kTileK != 0 || K > 65536) return W4A8_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const Schedule s = choose_schedule(M, N, K, dev < 0 ? 148 : num_sms(dev), true);
  if (tile_tokens) *tile_tokens = s.T;
  if (splits) *splits = s.splits;
  if (ctas) *ctas = s.ctas;
  return W4A8_OK;
}

int w4a8_get_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return W4A8_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return W4A8_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return W4A8_ERR_CUDA;
  return v;
}

int w4a8_debug_set_wait_budget(long long ns) {
  if (ns < -1 || ns > 10000000000ll) return W4A8_ERR_INVALID_ARG;
  g_wait_budget.store(ns, std::memory_order_relaxed);
  return W4A8_OK;
}

int w4a8_debug_timeout_probe(long long limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return W4A8_ERR_INVALID_ARG;
  timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>((unsigned long long)limit_ns);
  return cudaGetLastError() == cudaSuccess ? W4A8_OK : W4A8_ERR_CUDA;
}

}  // extern "C"
