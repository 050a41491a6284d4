// gemm.cuh -- the W4A8 GEMM for sm_100a: packed LQQ INT4 weights are
// dequantized to INT8 by CUDA-core warps straight into tensor memory (TMEM)
// and multiplied with INT8 activations by tcgen05.mma kind::i8 (INT32
// accumulators in TMEM), then a fused epilogue applies s_x[m] * s_w[n] and
// stores bf16 (or the exact INT32 accumulators).
//
// Method (review page "LiquidGEMM", pith.science verdict on arXiv
// 2509.01229): dequantization (q_u4 * s_u8 + a) XOR 0x80, two integer
// instructions per four weights after unpacking, never leaving UINT8
// (key_machinery; referee summary; referee minor 1, paper Sec. 5.3); the
// INT8 x INT8 tensor-core product with INT32 accumulation (lead); a
// producer / several-consumer pipeline that overlaps loading, CUDA-core
// dequantization and tensor-core MMA (key_machinery, "ImFP").
//
// The B200 design (not the page's Hopper design):
//   * MMA orientation: the 128 weight rows of a tile are the MMA's M
//     dimension and live in TMEM as the A operand (tcgen05.mma with A from
//     tensor memory); the T tokens of the tile are the MMA's N dimension
//     (B operand, shared memory, 128-byte swizzle, loaded by TMA).  The
//     dequantized weights therefore never touch shared memory: one
//     tcgen05.st per 32 weights and thread.
//   * Warp roles per CTA: warp 0 issues the copies (1-D bulk copy of a
//     packed weight tile + 2-D TMA of the activation tile), warp 1 issues
//     the MMAs, each through one elected lane of the converged warp; DQG
//     groups of 4 warps dequantize (thread = weight row = TMEM lane) and
//     then run the epilogue.
//   * Two rings.  SS shared-memory stages each hold one packed weight tile
//     and one activation tile (deep, to keep enough bytes in flight to
//     cover DRAM latency); AS TMEM slots of 32 columns each hold one
//     dequantized 128 x 128 weight tile (A operand).  Barriers: full[ss]
//     (copies landed), empty[ss] (the MMAs that read the stage completed),
//     dq[as] (A slot written), afree[as] (the MMAs that read the A slot
//     completed); the completions come from tcgen05.commit.
//   * Split-K for few output tiles (decode): the splits of one output tile
//     form a thread-block cluster.  Each CTA leaves its INT32 partial tile
//     in its own shared memory; after a cluster barrier every CTA sums one
//     slice of the tile over all partials through distributed shared memory
//     and applies the epilogue to it.  No global workspace, no atomics.
//   * Every wait is bounded (globaltimer); a wait that runs out records a
//     timeout in the device status word and all roles leave their loops,
//     wait for their own copies / MMAs in flight, free TMEM and return.
//   * W8 = true turns the same kernel into the W8A8 comparison point the
//     review page measures the method against (pith summary; forward
//     implication 3): plain INT8 weights [N][K] with one scale per channel,
//     loaded by 2-D TMA (128-byte swizzle) and read by the MMA straight from
//     shared memory; no dequantization, everything else (rings, split-K
//     cluster reduction, epilogue) unchanged.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace w4a8 {

enum : int { kModeStreamW = 1, kModeStoreY = 2 };

struct GemmParams {
  const uint8_t* tiles;   // packed weight tiles
  const float* s_w;       // packed per-channel scales [n_pad]
  const float* s_x;       // per-token scales [M] (bf16 output only)
  uint16_t* Y;            // [M][N] bf16 bits, or nullptr
  int32_t* acc;           // [M][N] int32, or nullptr
  int M, N, K, n_pad;
  int kt_total;           // K / 128
  int splits, kt_per_split;
  int n_tiles, m_tiles;
  // Tokens per tile actually used (the MMA's N): T, or in the runtime-width
  // instantiations of the 256-token tile a multiple of 16 below it (of 32
  // for CTA pairs) sized to the rows, so that no MMA work goes to rows that
  // do not exist.  The activation box is min(M, tn) rows (tn / 2 per CTA of
  // a pair).
  int tn;
  unsigned long long wait_limit_ns;
  const PackedHeader* hdr;  // checked against (N, K) before any store
  // Grouped GEMM (mixture-of-experts): rows [offsets[g], offsets[g+1]) of
  // Xq / Y belong to group g, whose packed weights start group_bytes * g
  // after `hdr`.  M is then the bound on rows per group, m_total the number
  // of rows of Xq / Y, and m_tiles the number of token-tile slots launched
  // (each slot takes the next token tile that holds rows, in group order).
  const int* offsets;     // [groups + 1] on the device, or nullptr (dense)
  size_t group_bytes;
  int m_total, groups;
  // Dense raster: tiles run through bands of `m_band` token tiles, channel
  // block by channel block, so that a wave of CTAs reuses both operands in
  // L2 (1 = channel blocks first).
  int m_band;
  // kModeStreamW: weight tiles are read by one token tile only (stream them
  // through L2 with evict-first; else normal priority).
  // kModeStoreY: without split-K, the bf16 tile is staged in shared memory
  // and written by one TMA tensor store through the second tensor map.
  int mode;
};
// (128 bytes: one more field measured 7% slower CTA-pair prefill launches)
static_assert(sizeof(GemmParams) <= 128, "kernel parameter block");

template <int T, int SS, int AS, int DQG, bool PUSH = false, bool W8 = false,
          bool PAIR = false, bool FUSED = false>
struct GemmCfg {
  // FUSED: the per-token activation quantization runs inside the GEMM (the
  // 16-token light ring, every k tile of a CTA resident at once)
  static_assert(!FUSED || (T == 16 && !W8 && !PAIR), "fused quantization: 16-token tiles");
  static_assert(T % 16 == 0 && T >= 16 && T <= 256, "MMA N for M=128");
  // PAIR: a 2-CTA cluster computes 256 channels x T tokens with CTA-pair
  // MMAs; each CTA holds its 128 channels (A and D in its tensor memory) and
  // loads half of the T tokens (B).
  static_assert(!PAIR || (T == 256 && !W8 && !PUSH), "CTA pairs use the 256-token tile");
  static_assert(AS <= SS, "the TMEM ring must not be deeper than the smem ring");
  // A dequantization group at k tile `it` waits for MMA(it - AS) on the A
  // slot's barrier.  Its own previous wait (tile it - DQG) guarantees
  // MMA(it - DQG - AS) done, which covers the slot's previous use
  // (it - 2 AS) only when AS >= DQG or there is one group; otherwise the
  // barrier can be two phases behind and the parity test passes on a stale
  // phase.
  static_assert(W8 || AS >= DQG || DQG == 1, "A slot ring too shallow for the dequant groups");
  static constexpr int kXBytes = (PAIR ? T / 2 : T) * kTileK;  // activation tile
  // weight stage: one packed LQQ tile, or a 128 x 128 INT8 tile (W8)
  static constexpr int kWBytes = W8 ? kTileN * kTileK : kTileBytes;
  static constexpr int kThreads = (2 + 4 * DQG) * 32;
  static constexpr int kA0 = T < 32 ? 32 : T;             // first A column
  static constexpr int kColsUsed = W8 ? kA0 : kA0 + 32 * AS;
  // a pair allocates all 512 columns, so both CTAs get column address 0
  static constexpr int kTmemCols = PAIR ? 512 : kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64
                                   : kColsUsed <= 128 ? 128 : kColsUsed <= 256 ? 256 : 512;
  static_assert(kColsUsed <= 512, "TMEM columns");
  // shared memory: x tiles | w tiles | barriers | misc | s_x cache
  static constexpr int kOffW = SS * kXBytes;
  static constexpr int kOffBar = kOffW + SS * kWBytes;
  static_assert(!W8 || (kOffW % 1024 == 0 && kWBytes % 1024 == 0),
                "128-byte-swizzled operand tiles start on 1024-byte boundaries");
  // stage barriers: weights landed, activations landed (not in the CTA-pair
  // form, which lands both on one), stage free; slot barriers; 3 more
  static constexpr int kNumBars = (PAIR ? 2 : 3) * SS + 2 * AS + 3 + (FUSED ? 1 : 0);
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kOffSx = kOffMisc + 16;
  // partial tiles of at most kPushMaxM tokens are pushed (remote atomic
  // adds) into the cluster leader's receive buffer; larger ones are gathered
  // from every CTA's stage buffers (remote atomics serialise at the leader)
  static constexpr bool kPush = PUSH;
  static constexpr int kPushMaxM = 8;
  static_assert(!PUSH || T == 16, "push reduction is for the 16-token tile");
  static constexpr int kOffRed = (kOffSx + 4 * T + 15) & ~15;
  static constexpr int kRedBytes = kPush ? T * kTileN * 4 : 0;
  // fused: the cluster-wide per-token absmax (fp32 bit patterns), then this
  // CTA's partial; the quantizing warps hold at most kFusedV float4 each
  static constexpr int kOffAmax = kOffRed + kRedBytes;
  static constexpr int kAmaxBytes = FUSED ? 2 * 4 * T : 0;
  static constexpr int kFusedV = 8;
  static constexpr int kSmemBytes = kOffAmax + kAmaxBytes + 1024;  // + alignment slack
  // the split-K partial tile reuses the pipeline buffers
  static_assert(T * kTileN * 4 <= kOffBar, "partial tile must fit the stage buffers");
};

// Dequantize four packed words (32 codes of one row, k order given by the
// packed layout) with the group's integer scale s and offset a into eight
// words of four INT8 values each: (code * s + a) XOR 0x80 per byte.
__device__ __forceinline__ void dequant_chunk(uint4 v, uint32_t s, uint32_t a4,
                                              uint32_t (&out)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t lo = w[j] & 0x0F0F0F0Fu;
    const uint32_t hi = (w[j] >> 4) & 0x0F0F0F0Fu;
    out[2 * j] = (lo * s + a4) ^ 0x80808080u;
    out[2 * j + 1] = (hi * s + a4) ^ 0x80808080u;
  }
}

// Ablation of the dequantization (the pages' argument for IMAD + XOR): each
// code unpacked on its own, code * s + min in signed 32-bit arithmetic,
// saturated to INT8 and packed back -- the "naive" route that has to guard
// against overflow.  Same results as dequant_chunk (the quantizer's bound
// means nothing saturates), many more instructions.
__device__ __forceinline__ void dequant_chunk_naive(uint4 v, int s, int mn, uint32_t (&out)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t packed = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int code = (int)((w[j] >> (8 * b + 4 * h)) & 0xFu);
        const int val = max(-128, min(127, code * s + mn));
        packed |= ((uint32_t)val & 0xFFu) << (8 * b);
      }
      out[2 * j + h] = packed;
    }
  }
}

constexpr int kClusterMax = 8;  // largest split-K cluster (portable cluster size)

// Kernel variants for the ablation study (the production kernel is 0).
enum : int {
  kVarDefault = 0,
  kVarNaiveDequant = 1,  // dequant_chunk_naive instead of IMAD + XOR
  kVarGroupIssuesMma = 2,  // the dequantization warpgroup issues the MMAs itself
};

// Two bf16 values (round to nearest even) packed low-first into 32 bits.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// One output: bf16(acc * (s_x * s_w)) in fp32 with a single rounding, or
// the exact INT32 accumulator.
__device__ __forceinline__ void store_out(const GemmParams& p, int m, int n, int32_t a,
                                          float sx, float sw) {
  if (p.Y) {
    const float y = (float)a * (sx * sw);
    p.Y[(size_t)m * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
  } else {
    p.acc[(size_t)m * p.N + n] = a;
  }
}

// All 32 lanes wait; the warp proceeds only if every lane saw the phase
// complete (keeps the .sync.aligned tcgen05 instructions warp-uniform).
template <bool CLUSTER = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity,
                                          volatile int* abort, uint64_t lim) {
  const bool ok = mbar_wait<CLUSTER>(bar, parity, abort, lim);
  return __all_sync(0xffffffffu, ok);
}

template <int T, int SS, int AS, int DQG, int MINB, bool PUSH, bool W8, int V, bool PAIR,
          bool RTN, bool FUSED>
__global__ void __launch_bounds__(GemmCfg<T, SS, AS, DQG, PUSH, W8, PAIR, FUSED>::kThreads, MINB)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x,
                     const __grid_constant__ CUtensorMap tmap_w,  // W8 only
                     const GemmParams p) {
  using C = GemmCfg<T, SS, AS, DQG, PUSH, W8, PAIR, FUSED>;
  // tokens per tile (MMA N): p.tn in the runtime-width instantiations,
  // else the compile-time T (which keeps the full-tile code as tight as it
  // was; a runtime width measured up to 20% slower on full tiles)
  const int TN = RTN ? p.tn : T;
  static_assert(PAIR || C::kTmemCols * MINB <= 512,
                "tensor-memory columns of the CTAs resident on one SM");
  static_assert(V != kVarGroupIssuesMma || (DQG == 1 && !W8),
                "the issuing warpgroup must see every k tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Each stage has two landing barriers, weights (bar_full) and activations
  // (bar_fullx): the weight tiles are prefetched before the preceding
  // kernel finishes, and their dequantization need not wait for the
  // activations, which only the MMAs read (decode: 11-18% per quantize +
  // GEMM pair).  The CTA-pair form (large M, nothing to prefetch early)
  // lands both on bar_full, which measured 3% faster there.
  constexpr bool kSplitLand = !PAIR;
  const uint32_t bar_full = sbase + C::kOffBar;     // + 8 ss
  const uint32_t bar_fullx = kSplitLand ? bar_full + 8 * SS : bar_full;  // + 8 ss
  const uint32_t bar_empty = bar_full + (kSplitLand ? 16 : 8) * SS;  // + 8 ss
  const uint32_t bar_dq = bar_empty + 8 * SS;       // + 8 as
  const uint32_t bar_afree = bar_dq + 8 * AS;       // + 8 as
  const uint32_t bar_acc = bar_afree + 8 * AS;
  const uint32_t bar_done = bar_acc + 8;  // every epilogue warp finished with TMEM
  const uint32_t bar_red = bar_done + 8;  // pushed partials landed (cluster leader)
  const uint32_t bar_amax = bar_red + 8;  // fused: every split's token absmax landed
  const bool push = C::kPush && p.splits > 1 && p.M <= C::kPushMaxM;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* ep_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 12);
  float* sx_s = reinterpret_cast<float*>(smem + C::kOffSx);

  // tile coordinates: the splits of a tile are consecutive blocks (one
  // cluster), then channel blocks, then token blocks (then groups)
  // A CTA pair (PAIR; no split-K) is two consecutive blocks covering
  // channel blocks 2j and 2j + 1 of the same token tile.
  const int rank = PAIR ? (int)cluster_ctarank() : 0;
  const int split = PAIR ? 0 : blockIdx.x % p.splits;
  const int tile = PAIR ? blockIdx.x >> 1 : blockIdx.x / p.splits;
  const int n_units = PAIR ? p.n_tiles >> 1 : p.n_tiles;  // channel blocks (pairs) per row
  int n_tile, m_slot;  // channel block; token tile (grouped: token-tile slot)
  if (p.offsets == nullptr && p.m_band > 1) {
    const int span = p.m_band * n_units;
    const int m_first = (tile / span) * p.m_band;
    const int rows = min(p.m_band, p.m_tiles - m_first);
    const int within = tile % span;
    n_tile = within / rows;
    m_slot = m_first + within % rows;
  } else {
    n_tile = tile % n_units;
    m_slot = tile / n_units;
  }
  if (PAIR) n_tile = 2 * n_tile + rank;
  const int kt0 = split * p.kt_per_split;
  const int kt1 = min(kt0 + p.kt_per_split, p.kt_total);
  const int nk = kt1 - kt0;
  const uint64_t lim = p.wait_limit_ns;
  // rows of this tile: row_base .. row_base + t_valid - 1 of Xq / Y
  int row_base, t_valid;
  const uint8_t* w_tiles = p.tiles;
  const float* w_scale = p.s_w;
  const PackedHeader* w_hdr = p.hdr;
  if (p.offsets == nullptr) {
    row_base = m_slot * TN;
    t_valid = min(TN, p.M - row_base);
  } else {
    // Grouped: the row offsets may be written by the preceding kernel.  Token
    // tile slot `a` is the a-th tile that holds rows, counting group by
    // group.  Every CTA checks every group's offsets, so a call with an
    // invalid group stores nothing.  All CTAs of a cluster (the splits of
    // one tile) take the same branch, so a slot without work leaves before
    // any cluster barrier.
    pdl_wait();
    int a = m_slot;
    int g = -1, m_tile = 0, r0 = 0, r1 = 0;
    bool bad = false;
    for (int q = 0; q < p.groups; ++q) {
      const int q0 = p.offsets[q], q1 = p.offsets[q + 1];
      if (q0 < 0 || q1 < q0 || q1 > p.m_total || q1 - q0 > p.M) {
        bad = true;
        break;
      }
      const int cnt = (q1 - q0 + TN - 1) / TN;
      if (g < 0) {
        if (a < cnt) {
          g = q;
          m_tile = a;
          r0 = q0;
          r1 = q1;
        } else {
          a -= cnt;
        }
      }
    }
    if (bad) {
      if (threadIdx.x == 0) record_status(kDevBadOffsets);
      return;
    }
    if (g < 0) return;
    row_base = r0 + m_tile * TN;
    t_valid = min(TN, r1 - row_base);
    w_tiles += p.group_bytes * g;
    w_scale = reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(w_scale) +
                                             p.group_bytes * g);
    w_hdr = reinterpret_cast<const PackedHeader*>(reinterpret_cast<const uint8_t*>(w_hdr) +
                                                  p.group_bytes * g);
  }

  // the host never launches these; stay safe anyway
  if (FUSED && (nk > SS || t_valid * nk * (kTileK / 4) > 64 * C::kFusedV)) {
    if (threadIdx.x == 0) record_status(kDevTimeout);
    return;
  }

  // Every warp reaches a CTA-wide barrier converged: an aligned barrier
  // reached by a warp in pieces (one lane late) can complete early and
  // leave a phase open that a later barrier then completes without waiting.
  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < SS; ++s) {
        mbar_init(bar_full + 8 * s, 1);
        // fused: the two quantizing warps arrive instead of a TMA
        if (kSplitLand) mbar_init(bar_fullx + 8 * s, FUSED ? 2 : 1);
        mbar_init(bar_empty + 8 * s, 1);
      }
      for (int a = 0; a < AS; ++a) {
        // the even CTA of a pair also counts the odd CTA's relayed arrival
        mbar_init(bar_dq + 8 * a, PAIR && rank == 0 ? 8 : 4);
        mbar_init(bar_afree + 8 * a, 1);
      }
      mbar_init(bar_acc, 1);
      mbar_init(bar_done, 4 * DQG);
      mbar_init(bar_red, 1);
      *abort_flag = lim == 0 ? 1 : 0;  // a wait budget of 0: abort before any wait
      if (lim == 0) record_status(kDevTimeout);
      fence_barrier_init();
      // push reduction: the leader's receive barrier completes when every
      // other split's partial (t_valid x 128 INT32 adds) has landed
      if (push && split == 0)
        mbar_arrive_expect_tx(bar_red, (uint32_t)(p.splits - 1) * (uint32_t)t_valid * kTileN * 4u);
      if (FUSED) {
        // split-K: every split (this CTA included) sends one max per token;
        // one split: the quantizing warps arrive once the table is written
        mbar_init(bar_amax, 1);
        fence_barrier_init();
        if (p.splits > 1)
          mbar_arrive_expect_tx(bar_amax, (uint32_t)p.splits * (uint32_t)t_valid * 4u);
      }
      pdl_launch_dependents();
    }
    __syncwarp();
  } else if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), C::kTmemCols);
      tmem_relinquish();
    }
  }
  if (push && split == 0) {  // the leader's receive buffer starts at zero
    int4* red = reinterpret_cast<int4*>(smem + C::kOffRed);
    for (int i = threadIdx.x; i < C::kRedBytes / 16; i += C::kThreads)
      red[i] = make_int4(0, 0, 0, 0);
  }
  if (FUSED) {  // the absmax table starts at zero
    uint32_t* tab = reinterpret_cast<uint32_t*>(smem + C::kOffAmax);
    for (int i = threadIdx.x; i < 2 * T; i += C::kThreads) tab[i] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // every CTA of the cluster announces that its barriers and buffers are
  // initialised; the matching wait comes just before the first remote access
  if (push) cluster_arrive();
  if (PAIR) {
    // both CTAs' barriers exist before any cross-CTA arrival, and both
    // tensor-memory allocations start at the same column (the pair MMA
    // addresses both with one address); otherwise the pair does no work
    cluster_sync_all();
    const uint32_t other = (uint32_t)dsmem_ld_s32(
        dsmem_map(smem_u32(const_cast<uint32_t*>(tmem_slot)), (uint32_t)(rank ^ 1)));
    if (other != tmem && threadIdx.x == 0) {
      record_status(kDevTimeout);
      *abort_flag = 1;
    }
    __syncthreads();
  }

  // -------------------------------------- fused activation quantization
  // Warps 0 and 1 (idle until the MMAs can start) quantize this CTA's k
  // range of the fp32 activations straight into the stages' token tiles:
  // the per-token absmax over the CTA's range is combined across the
  // split-K cluster by an asynchronous max into every CTA's table, then
  // s_x = absmax / 127 and codes rint(x / s_x) clamped to +-127 -- the rule
  // and the arithmetic of act_quant_kernel, so the codes are the same.  The
  // tiles are written in the 128-byte-swizzled layout the TMA would have
  // produced (16-byte chunk c of token row t at chunk c ^ (t mod 8)).
  auto fused_quant = [&]() {
    const int at = warp * 32 + lane;           // 0 .. 63
    const float* X = p.s_x;                    // fused: fp32 activations [M][K]
    const int k_lo = kt0 * kTileK;
    // float4 of one row in this CTA's k range (a multiple of 32), and of
    // the whole slice; element f is float4 f % n4 of row f / n4, and the 32
    // elements a warp holds for one j belong to one row
    const int n4 = nk * (kTileK / 4);
    const int total4 = t_valid * n4;  // <= 64 * C::kFusedV (host-checked)
    uint32_t* part = reinterpret_cast<uint32_t*>(smem + C::kOffAmax) + T;  // CTA absmax [T]
    const uint32_t tab = sbase + C::kOffAmax;
    pdl_wait();  // X is produced by the preceding kernel
    // every load of the slice in flight at once; the values stay in
    // registers for the quantization below
    float4 xv[C::kFusedV];
#pragma unroll
    for (int j = 0; j < C::kFusedV; ++j) {
      const int f = at + 64 * j;
      if (f < total4) {
        const int t = f / n4;
        xv[j] = __ldg(reinterpret_cast<const float4*>(X + (size_t)(row_base + t) * p.K + k_lo) +
                      (f - t * n4));
      } else {
        xv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int j = 0; j < C::kFusedV; ++j) {
      const int f0 = 64 * j + 32 * warp;  // warp-uniform
      if (f0 < total4) {
        const float m = warp_max(absmax4(xv[j]));
        if (lane == 0) atomicMax(part + f0 / n4, __float_as_uint(m));
      }
    }
    named_bar_sync(2, 64);
    if (p.splits == 1) {
      // one CTA: the partials are the row maxima; one local arrive (no
      // cluster addressing in a launch without clusters)
      if (at < t_valid) reinterpret_cast<uint32_t*>(smem + C::kOffAmax)[at] = part[at];
      named_bar_sync(2, 64);
      if (at == 0) mbar_arrive(bar_amax);  // release: the epilogue reads the table
    } else {
      if (push) cluster_wait();  // every CTA's table and barrier are initialised
      if (at < t_valid) {
        const uint32_t v = part[at];
        for (int q = 0; q < p.splits; ++q)
          dsmem_red_async_max_u32(dsmem_map(tab + 4u * (uint32_t)at, (uint32_t)q), v,
                                  dsmem_map(bar_amax, (uint32_t)q));
      }
      // (on a timeout the abort flag is set; no barrier below waits on these warps)
      if (!warp_wait<true>(bar_amax, 0, abort_flag, lim)) return;
    }
    const uint32_t* amax = reinterpret_cast<const uint32_t*>(smem + C::kOffAmax);
#pragma unroll
    for (int j = 0; j < C::kFusedV; ++j) {
      const int f = at + 64 * j;
      if (f < total4) {
        const int t = f / n4, i = f - t * n4;
        const float sc = __fdiv_rn(__uint_as_float(amax[t]), 127.0f);
        // float4 i of the row: k tile i / 32, 16-byte chunk (i / 4) % 8,
        // word i % 4 of the chunk
        const int it = i >> 5, c = (i >> 2) & 7;
        sts32(sbase + it * C::kXBytes + t * 128 + ((c ^ (t & 7)) << 4) + 4 * (i & 3),
              quant4(xv[j], sc));
      }
    }
    fence_proxy_async_smem();  // the tiles above, seen by the MMA (async proxy)
    __syncwarp();
    if (lane == 0)
      for (int it = 0; it < nk; ++it) mbar_arrive(bar_fullx + 8 * it);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop and waits; one elected lane issues the
    // copies (a converged warp issues these single-thread instructions much
    // faster than a lone diverged lane).
    const bool leader = elect_one();
    // bytes landing on a stage's two barriers: the weight tile, and the
    // activation box
    const uint32_t x_bytes = (uint32_t)(PAIR ? TN / 2 : min(p.M, TN)) * kTileK;
    const uint32_t tx_w = kSplitLand ? C::kWBytes : C::kWBytes + x_bytes;
    const uint32_t tx_x = x_bytes;
    if (leader) {
      if (!FUSED) prefetch_tensormap(&tmap_x);  // (the fused form has no tensor maps)
      if (W8 || (p.mode & kModeStoreY)) prefetch_tensormap(&tmap_w);
    }
    const uint64_t pol =
        (p.mode & kModeStreamW) ? l2_policy_evict_first() : l2_policy_evict_normal();
    const uint8_t* wsrc = W8 ? nullptr
                             : w_tiles + ((size_t)n_tile * p.kt_total + kt0) * kTileBytes;
    // one weight stage: a bulk copy of the packed tile, or a TMA box of
    // 128 channels x 128 k of the INT8 matrix
    auto load_w = [&](int it, int s) {
      if (W8)
        tma_load_2d(sbase + C::kOffW + s * C::kWBytes, &tmap_w, (kt0 + it) * kTileK,
                    n_tile * kTileN, bar_full + 8 * s);
      else
        bulk_g2s(sbase + C::kOffW + s * kTileBytes, wsrc + (size_t)it * kTileBytes,
                 kTileBytes, bar_full + 8 * s, pol);
    };
    int issued = 0;
    // The weights do not depend on the preceding kernel: the first ring's
    // worth of weight tiles is requested before waiting for it.
    const int pre = nk < SS ? nk : SS;
    if (leader) {
      for (int it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx(bar_full + 8 * it, tx_w);
        load_w(it, it);
      }
    }
    if (!FUSED) {
      pdl_wait();  // activations are produced by the preceding kernel
      if (leader) {
        for (int it = 0; it < pre; ++it) {
          if (kSplitLand) mbar_arrive_expect_tx(bar_fullx + 8 * it, tx_x);
          tma_load_2d(sbase + it * C::kXBytes, &tmap_x, (kt0 + it) * kTileK,
                      row_base + rank * (TN / 2), bar_fullx + 8 * it);
        }
      }
    }
    issued = pre;
    __syncwarp();
    if (FUSED) fused_quant();
    for (int it = pre; it < nk; ++it) {
      const int s = it % SS;
      const uint32_t ph = (it / SS) & 1;
      if (!warp_wait(bar_empty + 8 * s, ph ^ 1, abort_flag, lim)) break;
      if (leader) {
        mbar_arrive_expect_tx(bar_full + 8 * s, tx_w);
        load_w(it, s);
        if (!FUSED) {  // (fused calls have every k tile resident: no refills)
          if (kSplitLand) mbar_arrive_expect_tx(bar_fullx + 8 * s, tx_x);
          tma_load_2d(sbase + s * C::kXBytes, &tmap_x, (kt0 + it) * kTileK,
                      row_base + rank * (TN / 2), bar_fullx + 8 * s);
        }
      }
      __syncwarp();
      issued = it + 1;
    }
    if (*abort_flag) {
      // let the copies already issued land before the CTA goes away
      for (int it = issued - SS < 0 ? 0 : issued - SS; it < issued; ++it) {
        mbar_wait(bar_full + 8 * (it % SS), (it / SS) & 1, nullptr, kDrainLimitNs);
        if (kSplitLand)
          mbar_wait(bar_fullx + 8 * (it % SS), (it / SS) & 1, nullptr, kDrainLimitNs);
      }
    }
    __syncwarp();  // reconverge before any CTA- or cluster-wide barrier
  } else if (warp == 1 && PAIR) {
    // ------------------------------------------- MMA issuer of a CTA pair
    // The even CTA issues every MMA for both: it waits for both CTAs'
    // weight slots (its dq barrier counts one arrival relayed from the odd
    // CTA, which also means that CTA's token half of the stage has landed)
    // and for its own stage; the completions arrive on the barriers of both
    // CTAs.  In the odd CTA this warp is the relay: once its four
    // dequantization warps have arrived locally on a slot it makes the one
    // cluster-scope release arrive on the even CTA's barrier, keeping that
    // fence off the dequantization warps.
    if (rank == 0) {
      const bool leader = elect_one();
      const uint32_t idesc = idesc_i8(256, TN);
      for (int it = 0; it < nk; ++it) {
        const int s = it % SS, a = it % AS;
        if (!warp_wait<true>(bar_dq + 8 * a, (it / AS) & 1, abort_flag, lim)) break;
        if (!warp_wait(bar_fullx + 8 * s, (it / SS) & 1, abort_flag, lim)) break;
        tc_fence_after();
        if (leader) {
          const uint64_t bdesc = smem_desc_sw128(sbase + s * C::kXBytes);
          const uint32_t a_tmem = tmem + C::kA0 + 32 * a;
#pragma unroll
          for (int kk = 0; kk < kTileK / 32; ++kk)
            mma_i8_ts_pair(tmem, a_tmem + 8 * kk, bdesc + (uint64_t)(2 * kk), idesc,
                           (it | kk) != 0);
          tc_commit_pair(bar_empty + 8 * s);
          tc_commit_pair(bar_afree + 8 * a);
        }
        __syncwarp();
      }
      if (leader) tc_commit_pair(bar_acc);  // also on abort: tracks every MMA issued
      __syncwarp();
    }
  } else if (warp == 1 && V != kVarGroupIssuesMma) {
    // ---------------------------------------------------------- MMA issuer
    // Whole warp waits, one elected lane issues the MMAs and commits.
    if (FUSED) fused_quant();
    const bool leader = elect_one();
    const uint32_t idesc = idesc_i8(128, TN);
    for (int it = 0; it < nk; ++it) {
      const int s = it % SS, a = it % AS;
      // the weights reach the MMA through the dequantized slot (dq), except
      // in the W8A8 form, which reads the stage's INT8 weight tile directly
      if (!W8 && !warp_wait(bar_dq + 8 * a, (it / AS) & 1, abort_flag, lim)) break;
      if (W8 && !warp_wait(bar_full + 8 * s, (it / SS) & 1, abort_flag, lim)) break;
      if (!warp_wait(bar_fullx + 8 * s, (it / SS) & 1, abort_flag, lim)) break;
      tc_fence_after();
      if (leader) {
        const uint64_t bdesc = smem_desc_sw128(sbase + s * C::kXBytes);
        if (W8) {
          // both operands in shared memory; +32 bytes of k per instruction
          const uint64_t adesc = smem_desc_sw128(sbase + C::kOffW + s * C::kWBytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / 32; ++kk)
            mma_i8_ss(tmem, adesc + (uint64_t)(2 * kk), bdesc + (uint64_t)(2 * kk), idesc,
                      (it | kk) != 0);
          tc_commit(bar_empty + 8 * s);
        } else {
          const uint32_t a_tmem = tmem + C::kA0 + 32 * a;
#pragma unroll
          for (int kk = 0; kk < kTileK / 32; ++kk)
            mma_i8_ts(tmem, a_tmem + 8 * kk, bdesc + (uint64_t)(2 * kk), idesc,
                      (it | kk) != 0);
          tc_commit(bar_empty + 8 * s);
          tc_commit(bar_afree + 8 * a);
        }
      }
      __syncwarp();
    }
    if (leader) tc_commit(bar_acc);  // also on abort: tracks every MMA issued
    __syncwarp();
  } else if (warp >= 2) {
    // --------------------------------------------- dequantization warps
    const int dg = (warp - 2) / 4;         // dequant group
    const int quarter = warp & 3;          // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;     // weight row in the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int n = n_tile * kTileN + r;
    // loads needed only by the epilogue, issued before the main loop so
    // their latency is hidden
    const float swn = (p.Y && n < p.N) ? __ldg(w_scale + n) : 0.0f;  // no scales for INT32 output
    bool hdr_ok = true;
    if (!W8 && warp == 2 && lane == 0)
      hdr_ok = w_hdr->magic == kMagic && w_hdr->N == p.N && w_hdr->K == p.K;
    for (int it = dg; !W8 && it < nk; it += DQG) {
      const int s = it % SS, a = it % AS;
      // First the A slot's previous contents must be consumed (its MMAs
      // done).  That also settles the parity wait on the stage's full
      // barrier: a group skips the other group's iterations and could
      // otherwise reach round k of a stage while round k-1's copies are
      // still in flight, when the barrier's last completed phase (k-2) has
      // the parity of k.  MMA(it - AS) done implies every stage round
      // before this one has landed, because AS <= SS.
      if (!warp_wait(bar_afree + 8 * a, ((it / AS) & 1) ^ 1, abort_flag, lim)) break;
      if (!warp_wait(bar_full + 8 * s, (it / SS) & 1, abort_flag, lim)) break;
      // (in the CTA-pair form bar_full also covers the token half, which the
      // odd CTA's arrival on the even one's slot barrier thereby implies)
      tc_fence_after();
      // all shared-memory reads first (independent), then the arithmetic,
      // then one 32-column TMEM store of this row's 128 dequantized weights
      const uint32_t wbase = sbase + C::kOffW + s * kTileBytes;
      uint4 v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = lds128(wbase + (c * kTileN + r) * 16);
      const uint32_t prm = lds32(wbase + kCodeBytes + 4 * r);
      uint32_t out[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t sh = (c < 2) ? 0 : 16;
        const uint32_t sc = (prm >> sh) & 0xFFu;
        if (V == kVarNaiveDequant) {
          const int mn = (int)((prm >> (sh + 8)) & 0xFFu) - 128;
          dequant_chunk_naive(v[c], (int)sc, mn, *reinterpret_cast<uint32_t(*)[8]>(out + 8 * c));
        } else {
          const uint32_t a4 = ((prm >> (sh + 8)) & 0xFFu) * 0x01010101u;
          dequant_chunk(v[c], sc, a4, *reinterpret_cast<uint32_t(*)[8]>(out + 8 * c));
        }
      }
      tmem_st_x32(lane_base + C::kA0 + 32 * a, out);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && rank != 0)
          mbar_arrive_remote_relaxed(dsmem_map(bar_dq + 8 * a, 0));
        else
          mbar_arrive(bar_dq + 8 * a);
      }
      if (V == kVarGroupIssuesMma && warp == 2) {
        // ablation: the first warp of the (single) dequantization group
        // issues this k tile's MMAs once all four quarters are in TMEM
        if (!warp_wait(bar_dq + 8 * a, (it / AS) & 1, abort_flag, lim)) break;
        if (!warp_wait(bar_fullx + 8 * s, (it / SS) & 1, abort_flag, lim)) break;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t bdesc = smem_desc_sw128(sbase + s * C::kXBytes);
          const uint32_t a_tmem = tmem + C::kA0 + 32 * a;
#pragma unroll
          for (int kk = 0; kk < kTileK / 32; ++kk)
            mma_i8_ts(tmem, a_tmem + 8 * kk, bdesc + (uint64_t)(2 * kk), idesc_i8(128, TN),
                      (it | kk) != 0);
          tc_commit(bar_empty + 8 * s);
          tc_commit(bar_afree + 8 * a);
        }
        __syncwarp();
      }
    }
    if (V == kVarGroupIssuesMma && warp == 2) {
      if (elect_one()) tc_commit(bar_acc);  // also on abort: tracks every MMA issued
      __syncwarp();
    }

    // -------------------------------------------------------- epilogue
    const int nthr = 128 * DQG;
    const int et = threadIdx.x - 64;  // epilogue thread index
    pdl_wait();  // s_x and the outputs are ordered after the preceding kernel
    if (p.Y) {
      if (FUSED) {
        // s_x from the cluster's absmax table (p.s_x holds the fp32 input)
        warp_wait<true>(bar_amax, 0, abort_flag, lim);
        const uint32_t* amax = reinterpret_cast<const uint32_t*>(smem + C::kOffAmax);
        for (int i = et; i < T; i += nthr)
          sx_s[i] = i < t_valid ? __fdiv_rn(__uint_as_float(amax[i]), 127.0f) : 0.0f;
      } else {
        for (int i = et; i < T; i += nthr) sx_s[i] = i < t_valid ? p.s_x[row_base + i] : 0.0f;
      }
    }
    warp_wait(bar_acc, 0, abort_flag, lim);
    tc_fence_after();
    // one thread turns the abort flag into a value every epilogue thread
    // reads between the same two barriers, so the branches below are uniform
    named_bar_sync(1, nthr);
    if (warp == 2 && lane == 0) {
      if (!hdr_ok) record_status(kDevBadPacked);
      *ep_flag = (*abort_flag || !hdr_ok) ? 0 : 1;
    }
    __syncwarp();
    named_bar_sync(1, nthr);
    if (*ep_flag) {
      if (!W8 && p.splits == 1 && (p.mode & kModeStoreY)) {
        // stage the bf16 tile as [token][128 channels] in the (free) stage
        // buffers, then one thread writes it with a TMA tensor store; rows
        // past M and channels past N are clipped by the store (only the
        // 16-column groups holding valid tokens are read from TMEM, here and
        // below: a 256-token tile at M = 128 carries 128)
        const uint32_t ystage = sbase;
        for (int j = dg; j < T / 16 && 16 * j < t_valid; j += DQG) {
          uint32_t v[16];
          tmem_ld_x16(lane_base + 16 * j, v);
          tmem_wait_ld();
          // two tokens per conversion instruction (the staging is bound by
          // its per-value work: 2-3% faster prefill than one at a time)
#pragma unroll
          for (int t = 0; t < 16; t += 2) {
            const int tt = 16 * j + t;
            const __nv_bfloat162 h =
                __floats2bfloat162_rn((float)(int32_t)v[t] * (sx_s[tt] * swn),
                                      (float)(int32_t)v[t + 1] * (sx_s[tt + 1] * swn));
            const uint32_t w = *reinterpret_cast<const uint32_t*>(&h);
            sts16(ystage + (uint32_t)(tt * kTileN + r) * 2u, (unsigned short)(w & 0xFFFFu));
            sts16(ystage + (uint32_t)((tt + 1) * kTileN + r) * 2u, (unsigned short)(w >> 16));
          }
        }
        fence_proxy_async_smem();  // the stores above, seen by the TMA engine
        named_bar_sync(1, nthr);
        if (threadIdx.x == 64) {
          tma_store_2d(&tmap_w, n_tile * kTileN, row_base, ystage);
          bulk_commit_group();
          bulk_wait_group_all();
        }
        __syncwarp();
      } else if (p.splits == 1) {
        for (int j = dg; j < T / 16 && 16 * j < t_valid; j += DQG) {
          uint32_t v[16];
          tmem_ld_x16(lane_base + 16 * j, v);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const int tt = 16 * j + t;
              if (tt < t_valid) store_out(p, row_base + tt, n, (int32_t)v[t], sx_s[tt], swn);
            }
          }
        }
      } else if (!push) {
        // partial tile -> own shared memory, token-major: part[t][r]
        // (the pipeline buffers are free: every copy landed and every MMA
        // that read them completed)
        int32_t* part = reinterpret_cast<int32_t*>(smem);
        for (int j = dg; j < T / 16 && 16 * j < t_valid; j += DQG) {
          uint32_t v[16];
          tmem_ld_x16(lane_base + 16 * j, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) part[(16 * j + t) * kTileN + r] = (int32_t)v[t];
        }
      }
    }
    if (push) {
      // split-K by pushing: the other CTAs add their partials into the
      // leader's receive buffer and arrive on its barrier; the leader adds
      // its own partial and runs the epilogue
      cluster_wait();
      const uint32_t red = sbase + C::kOffRed;
      if (split != 0) {
        // Every byte the leader expects is sent, zeros after an abort, so
        // the leader's wait always ends and it never leaves while adds are
        // still landing in its shared memory.
        const uint32_t red0 = dsmem_map(red, 0);
        const uint32_t bar0 = dsmem_map(bar_red, 0);
        const bool live = *ep_flag != 0;  // uniform over the CTA
        for (int j = dg; j < T / 16; j += DQG) {
          if (16 * j >= t_valid) break;
          uint32_t v[16];
          if (live) {
            tmem_ld_x16(lane_base + 16 * j, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int t = 0; t < 16; ++t) v[t] = 0;
          }
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (16 * j + t < t_valid)
              dsmem_red_async_add_s32(red0 + 4u * (uint32_t)((16 * j + t) * kTileN + r),
                                      (int32_t)v[t], bar0);
        }
        __syncwarp();
      } else {
        // remote arrivals (cluster scope); the full budget even after this
        // CTA's own abort: the other splits' adds land in its memory
        warp_wait<true>(bar_red, 0, nullptr, kDrainLimitNs);
        if (*ep_flag) {
          const int32_t* rb = reinterpret_cast<const int32_t*>(smem + C::kOffRed);
          for (int j = dg; j < T / 16; j += DQG) {
            if (16 * j >= t_valid) break;
            uint32_t v[16];
            tmem_ld_x16(lane_base + 16 * j, v);
            tmem_wait_ld();
            if (n < p.N) {
#pragma unroll
              for (int t = 0; t < 16; ++t) {
                const int tt = 16 * j + t;
                if (tt < t_valid)
                  store_out(p, row_base + tt, n, (int32_t)v[t] + rb[tt * kTileN + r], sx_s[tt],
                            swn);
              }
            }
          }
        }
      }
    }
    __syncwarp();
  }

  if (p.splits > 1 && !push) {
    // ---------------------- split-K by gathering partials over the cluster
    cluster_sync_all();  // every partial (and every split's ep_flag) is in shared memory
    // a split that aborted wrote no partial: store nothing unless every
    // split of the cluster completed (one remote read per split and warp)
    bool all_ok = false;
    if (warp >= 2) {
      int ok = 1;
      if (lane == 0) {
        const uint32_t epa = sbase + C::kOffMisc + 12;
        int got[kClusterMax];
#pragma unroll
        for (int q = 0; q < kClusterMax; ++q)
          got[q] = q < p.splits ? dsmem_ld_s32(dsmem_map(epa, (uint32_t)q)) : 1;
#pragma unroll
        for (int q = 0; q < kClusterMax; ++q) ok &= got[q] != 0;
      }
      all_ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
    }
    if (warp >= 2 && all_ok) {
      const int nthr = 128 * DQG;
      const int et = threadIdx.x - 64;
      const int total = t_valid * kTileN;
      // slices of whole 16-byte groups (4 consecutive channels of a token)
      const int per = ((total + p.splits - 1) / p.splits + 3) & ~3;
      const int e0 = split * per, e1 = min(total, e0 + per);
      const uint32_t part0 = sbase;
      // whole-group vector stores when every output row starts 16 bytes
      // aligned (N a multiple of 4 for bf16 8-byte stores, of 4 for INT32
      // 16-byte stores) and the buffer itself is aligned
      const bool vec_out = (p.N % 4) == 0 &&
                           (p.Y ? (reinterpret_cast<uintptr_t>(p.Y) & 7) == 0
                                : (reinterpret_cast<uintptr_t>(p.acc) & 15) == 0);
      constexpr int kBatch = 2;  // groups in flight per thread and round
      for (int eb = e0 + 4 * et; eb < e1; eb += 4 * nthr * kBatch) {
        // issue every remote load of the round (all splits) before using
        // any of them: the loads are in flight together, not one round trip
        // per split
        int4 got[kClusterMax][kBatch];
#pragma unroll
        for (int q = 0; q < kClusterMax; ++q) {
#pragma unroll
          for (int b = 0; b < kBatch; ++b) {
            const int e = eb + 4 * nthr * b;
            got[q][b] = (q < p.splits && e < e1)
                            ? dsmem_ld_v4(dsmem_map(part0 + 4u * (uint32_t)e, (uint32_t)q))
                            : make_int4(0, 0, 0, 0);
          }
        }
        int4 acc4[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          acc4[b] = got[0][b];
#pragma unroll
          for (int q = 1; q < kClusterMax; ++q) {
            acc4[b].x += got[q][b].x;
            acc4[b].y += got[q][b].y;
            acc4[b].z += got[q][b].z;
            acc4[b].w += got[q][b].w;
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int e = eb + 4 * nthr * b;
          if (e >= e1) continue;
          const int t = e / kTileN, r2 = e % kTileN;
          const int n2 = n_tile * kTileN + r2;
          // packed s_w is padded to whole channel blocks, so the 4-wide load
          // is in bounds; the W8 scales are exactly N long
          float4 sw4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (p.Y) {
            if (!W8) {
              sw4 = __ldg(reinterpret_cast<const float4*>(w_scale + n2));
            } else {
              sw4.x = __ldg(w_scale + n2);
              if (n2 + 1 < p.N) sw4.y = __ldg(w_scale + n2 + 1);
              if (n2 + 2 < p.N) sw4.z = __ldg(w_scale + n2 + 2);
              if (n2 + 3 < p.N) sw4.w = __ldg(w_scale + n2 + 3);
            }
          }
          const int32_t av[4] = {acc4[b].x, acc4[b].y, acc4[b].z, acc4[b].w};
          const float swv[4] = {sw4.x, sw4.y, sw4.z, sw4.w};
          const size_t o = (size_t)(row_base + t) * p.N + n2;
          if (vec_out && n2 + 4 <= p.N) {
            // the group's 4 channels are contiguous in the output row
            if (p.Y) {
              const float sx = sx_s[t];
              uint2 w;
              w.x = pack_bf16x2((float)av[0] * (sx * swv[0]), (float)av[1] * (sx * swv[1]));
              w.y = pack_bf16x2((float)av[2] * (sx * swv[2]), (float)av[3] * (sx * swv[3]));
              *reinterpret_cast<uint2*>(p.Y + o) = w;
            } else {
              *reinterpret_cast<int4*>(p.acc + o) = acc4[b];
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (n2 + i < p.N) store_out(p, row_base + t, n2 + i, av[i], sx_s[t], swv[i]);
          }
        }
      }
    }
    __syncwarp();
    cluster_sync_all();  // no CTA leaves while another still reads its partials
  }

  // ------------------------------------------------------------ teardown
  // Each epilogue warp reports that it no longer touches TMEM; the warp that
  // frees TMEM waits for all of them (and, after an abort, for every MMA).
  if (warp >= 2) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_done);
  }
  // pairs with the arrive at set-up (the fused quantizing warps waited already)
  if (push && warp < 2 && !FUSED) cluster_wait();
  if (warp == 1) {
    // after an abort the commit on bar_acc tracks every MMA issued; each
    // completes within microseconds, so with the full drain budget this wait
    // ends with the MMAs done and tensor memory is never freed under them
    warp_wait(bar_done, 0, nullptr, kDrainLimitNs);
    if (*abort_flag) warp_wait(bar_acc, 0, nullptr, kDrainLimitNs);
    // fused split-K: every split's absmax (sent unconditionally) has landed
    if (FUSED && p.splits > 1) warp_wait<true>(bar_amax, 0, nullptr, kDrainLimitNs);
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, C::kTmemCols);
    else
      tmem_dealloc(tmem, C::kTmemCols);
  }
  __syncwarp();
  __syncthreads();
  // neither CTA of a pair leaves while the other may still arrive on its
  // barriers
  if (PAIR) cluster_sync_all();
}

}  // namespace w4a8
