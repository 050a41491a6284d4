// gemm_pp.cuh -- the persistent CTA-pair form of the W4A8 GEMM for large M
// (prefill): the same method and per-k-tile pipeline as w4a8_gemm_kernel's
// CTA-pair form (packed LQQ tiles dequantized into tensor memory by CUDA-core
// warps, (code * s_u8 + a) XOR 0x80 per byte -- review page "LiquidGEMM",
// key_machinery; INT8 x INT8 tcgen05 MMAs accumulating in INT32 -- lead),
// rearranged so that a tile's epilogue overlaps the next tile's main loop:
//
//   * The grid is one CTA pair per two SMs.  Each pair walks the output
//     tiles (256 channels x TW tokens) tile = pair, pair + pairs, ... in the
//     raster order of the dense launch (bands of token tiles).
//   * Two accumulators of TW columns live in tensor memory next to the AS
//     weight slots (2 TW + 32 AS = 512 columns with TW = 192, AS = 4).  The
//     MMA warp fills accumulator i % 2 while dedicated epilogue warps drain
//     the other one: tcgen05.ld, fp32 epilogue, one bf16 rounding, staging
//     in shared memory, one TMA tensor store per tile.  The epilogue warps
//     release an accumulator (an mbarrier the MMA warp waits on before its
//     first MMA into it) as soon as their loads of it completed.
//   * The copy, dequantization and MMA rings run on without a break between
//     tiles: their barrier phases follow a k-tile counter over all of the
//     CTA's tiles, so the next tile's copies and dequantization start while
//     the previous tile's MMAs finish and its epilogue runs.
//   * Everything else is the CTA-pair form's: each CTA dequantizes its own
//     128 channels into its own tensor memory (A) and loads half of the
//     tokens (B); the even CTA issues the pair MMAs (M = 256) and their
//     completions arrive on both CTAs' barriers; the odd CTA's arrivals on
//     the even CTA's barriers are relaxed cluster-scope arrivals made after
//     its own tensor-memory stores (or loads) completed.
//   * Every wait is bounded; after an abort every role leaves its loop, the
//     copies issued land, a final commit covers every MMA issued, and only
//     then is tensor memory freed.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "gemm.cuh"
#include "layout.cuh"
#include "ptx.cuh"

namespace w4a8 {

struct PpParams {
  const uint8_t* tiles;   // packed weight tiles
  const float* s_w;       // packed per-channel scales [n_pad]
  const float* s_x;       // per-token scales [M] (bf16 output)
  int32_t* acc;           // [M][N] int32, or nullptr (bf16 output through tmap_y)
  const PackedHeader* hdr;
  int M, N, K;
  int kt_total;           // K / 128
  int n_pairs;            // channel-block pairs (N padded to 256)
  int m_tiles;            // token tiles of TW
  int m_band;             // token tiles per raster band
  unsigned long long wait_limit_ns;
};

template <int TW, int SS, int AS>
struct PpCfg {
  static_assert(TW % 32 == 0 && TW >= 64 && TW <= 224, "token tile: a multiple of 32");
  static_assert(2 * TW + 32 * AS <= 512, "two accumulators and the weight slots in TMEM");
  static_assert(AS >= 2 && AS <= SS, "weight slots");
  static constexpr int kDQG = 2;                         // dequantization groups
  static constexpr int kEpiWarps = 4;                    // one per TMEM lane quarter
  static constexpr int kThreads = (2 + 4 * kDQG + kEpiWarps) * 32;
  static constexpr int kFirstEpiWarp = 2 + 4 * kDQG;
  static constexpr int kXBytes = (TW / 2) * kTileK;      // this CTA's half of the tokens
  static constexpr int kStageBytes = kTileBytes + kXBytes;
  static constexpr int kOffX = 0;                        // SS activation halves
  static constexpr int kOffW = SS * kXBytes;             // SS packed weight tiles
  static constexpr int kOffY = kOffW + SS * kTileBytes;  // bf16 staging [TW][128]
  static constexpr int kYBytes = TW * kTileN * 2;
  static constexpr int kOffSx = kOffY + kYBytes;         // s_x of the tile [TW]
  static constexpr int kOffBar = (kOffSx + 4 * TW + 7) & ~7;
  // full[SS], empty[SS], dq[AS], afree[AS], acc[2], accfree[2], fin, done
  static constexpr int kNumBars = 2 * SS + 2 * AS + 6;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static_assert(kOffX % 1024 == 0 && kXBytes % 1024 == 0, "swizzled token tiles");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
  static constexpr int kA0 = 2 * TW;                     // first weight-slot column
};

template <int TW, int SS, int AS>
__global__ void __launch_bounds__(PpCfg<TW, SS, AS>::kThreads, 1)
    w4a8_gemm_pp_kernel(const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_y, const PpParams p) {
  using C = PpCfg<TW, SS, AS>;
  constexpr int DQG = C::kDQG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, pairs = gridDim.x >> 1;
  const int tiles_total = p.m_tiles * p.n_pairs;
  const int nk = p.kt_total;
  const uint64_t lim = p.wait_limit_ns;

  const uint32_t bar_full = sbase + C::kOffBar;           // + 8 s: stage landed
  const uint32_t bar_empty = bar_full + 8 * SS;           // + 8 s: stage consumed
  const uint32_t bar_dq = bar_empty + 8 * SS;             // + 8 a: weight slot written
  const uint32_t bar_afree = bar_dq + 8 * AS;             // + 8 a: weight slot consumed
  const uint32_t bar_acc = bar_afree + 8 * AS;            // + 8 b: accumulator ready
  const uint32_t bar_accfree = bar_acc + 16;              // + 8 b: accumulator drained
  const uint32_t bar_fin = bar_accfree + 16;              // every MMA issued completed
  const uint32_t bar_done = bar_fin + 8;                  // every epilogue warp done
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  float* sx_s = reinterpret_cast<float*>(smem + C::kOffSx);

  // tile -> (channel-block pair, token tile): bands of m_band token tiles,
  // channel-block pairs within a band (the dense launch's raster)
  auto tile_coords = [&](int tile, int& n_pair, int& m_tile) {
    const int span = p.m_band * p.n_pairs;
    const int m_first = (tile / span) * p.m_band;
    const int rows = min(p.m_band, p.m_tiles - m_first);
    const int within = tile % span;
    n_pair = within / rows;
    m_tile = m_first + within % rows;
  };
  const int my_tiles = pair < tiles_total ? (tiles_total - pair + pairs - 1) / pairs : 0;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < SS; ++s) {
        mbar_init(bar_full + 8 * s, 1);
        mbar_init(bar_empty + 8 * s, 1);
      }
      for (int a = 0; a < AS; ++a) {
        mbar_init(bar_dq + 8 * a, rank == 0 ? 8 : 4);  // even CTA: both CTAs' warps
        mbar_init(bar_afree + 8 * a, 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar_acc + 8 * b, 1);
        mbar_init(bar_accfree + 8 * b, rank == 0 ? 2 * C::kEpiWarps : C::kEpiWarps);
      }
      mbar_init(bar_fin, 1);
      mbar_init(bar_done, C::kEpiWarps);
      *abort_flag = lim == 0 ? 1 : 0;  // a wait budget of 0: abort before any wait
      if (lim == 0) record_status(kDevTimeout);
      fence_barrier_init();
      pdl_launch_dependents();
    }
    __syncwarp();
  } else if (warp == 1) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // both CTAs' barriers exist before any cross-CTA arrival, and both
  // allocations start at the same column (the pair MMA addresses both with
  // one address); otherwise the pair does no work
  cluster_sync_all();
  {
    const uint32_t other = (uint32_t)dsmem_ld_s32(
        dsmem_map(smem_u32(const_cast<uint32_t*>(tmem_slot)), rank ^ 1u));
    if (other != tmem && threadIdx.x == 0) {
      record_status(kDevTimeout);
      *abort_flag = 1;
    }
    __syncthreads();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const bool leader = elect_one();
    if (leader) prefetch_tensormap(&tmap_x);
    pdl_wait();  // activations are produced by the preceding kernel
    const uint64_t pol = l2_policy_evict_normal();
    const uint32_t tx = (uint32_t)(kTileBytes + C::kXBytes);
    long g = 0;  // k tiles issued over all of this CTA's tiles
    for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
      int n_pair, m_tile;
      tile_coords(pair + i * pairs, n_pair, m_tile);
      const int n_tile = 2 * n_pair + (int)rank;
      const uint8_t* wsrc = p.tiles + (size_t)n_tile * p.kt_total * kTileBytes;
      const int row = m_tile * TW + (int)rank * (TW / 2);
      bool ok = true;
      for (int it = 0; it < nk; ++it, ++g) {
        const int s = (int)(g % SS);
        if (!warp_wait(bar_empty + 8 * s, (uint32_t)((g / SS) & 1) ^ 1u, abort_flag, lim)) {
          ok = false;
          break;
        }
        if (leader) {
          mbar_arrive_expect_tx(bar_full + 8 * s, tx);
          bulk_g2s(sbase + C::kOffW + s * kTileBytes, wsrc + (size_t)it * kTileBytes,
                   kTileBytes, bar_full + 8 * s, pol);
          tma_load_2d(sbase + C::kOffX + s * C::kXBytes, &tmap_x, it * kTileK, row,
                      bar_full + 8 * s);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
    if (*abort_flag) {
      // let the copies already issued land before the CTA goes away
      for (long h = g - SS < 0 ? 0 : g - SS; h < g; ++h)
        mbar_wait(bar_full + 8 * (int)(h % SS), (uint32_t)((h / SS) & 1), nullptr,
                  kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (even CTA only)
    if (rank == 0) {
      const bool leader = elect_one();
      const uint32_t idesc = idesc_i8(256, TW);
      long g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int b = i & 1;
        // both CTAs' epilogues drained this accumulator (tile i - 2)
        if (!warp_wait<true>(bar_accfree + 8 * b, (uint32_t)((i >> 1) & 1) ^ 1u, abort_flag,
                             lim))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * TW);
        for (int it = 0; it < nk; ++it, ++g) {
          const int s = (int)(g % SS), a = (int)(g % AS);
          if (!warp_wait<true>(bar_dq + 8 * a, (uint32_t)((g / AS) & 1), abort_flag, lim) ||
              !warp_wait(bar_full + 8 * s, (uint32_t)((g / SS) & 1), abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (leader) {
            const uint64_t bdesc = smem_desc_sw128(sbase + C::kOffX + s * C::kXBytes);
            const uint32_t a_tmem = tmem + C::kA0 + 32 * a;
#pragma unroll
            for (int kk = 0; kk < kTileK / 32; ++kk)
              mma_i8_ts_pair(d_tmem, a_tmem + 8 * kk, bdesc + (uint64_t)(2 * kk), idesc,
                             (it | kk) != 0);
            tc_commit_pair(bar_empty + 8 * s);
            tc_commit_pair(bar_afree + 8 * a);
          }
          __syncwarp();
        }
        if (ok && leader) tc_commit_pair(bar_acc + 8 * b);
        __syncwarp();
      }
      if (leader) tc_commit_pair(bar_fin);  // tracks every MMA issued (also on abort)
      __syncwarp();
    }
  } else if (warp < C::kFirstEpiWarp) {
    // --------------------------------------------- dequantization warps
    const int dg = (warp - 2) / 4;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // weight row in the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const long total = (long)my_tiles * nk;
    for (long g = dg; g < total; g += DQG) {
      const int s = (int)(g % SS), a = (int)(g % AS);
      // the slot's previous contents consumed (see w4a8_gemm_kernel: this
      // also settles the parity wait on the stage's full barrier)
      if (!warp_wait(bar_afree + 8 * a, (uint32_t)((g / AS) & 1) ^ 1u, abort_flag, lim)) break;
      if (!warp_wait(bar_full + 8 * s, (uint32_t)((g / SS) & 1), abort_flag, lim)) break;
      tc_fence_after();
      const uint32_t wbase = sbase + C::kOffW + s * kTileBytes;
      uint4 v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) v[c] = lds128(wbase + (c * kTileN + r) * 16);
      const uint32_t prm = lds32(wbase + kCodeBytes + 4 * r);
      uint32_t out[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t sh = (c < 2) ? 0 : 16;
        const uint32_t a4 = ((prm >> (sh + 8)) & 0xFFu) * 0x01010101u;
        dequant_chunk(v[c], (prm >> sh) & 0xFFu, a4, *reinterpret_cast<uint32_t(*)[8]>(out + 8 * c));
      }
      tmem_st_x32(lane_base + C::kA0 + 32 * a, out);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank != 0)
          mbar_arrive_remote_relaxed(dsmem_map(bar_dq + 8 * a, 0));
        else
          mbar_arrive(bar_dq + 8 * a);
      }
    }
  } else {
    // ---------------------------------------------------- epilogue warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // channel row in the tile = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int et = threadIdx.x - C::kFirstEpiWarp * 32;  // 0 .. 127
    const bool ystore = p.acc == nullptr;
    const uint32_t ystage = sbase + C::kOffY;
    volatile int* ep_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);
    // (every epilogue thread reads the header: the outcome is uniform)
    const bool hdr_ok = p.hdr->magic == kMagic && p.hdr->N == p.N && p.hdr->K == p.K;
    if (et == 0 && !hdr_ok) record_status(kDevBadPacked);
    pdl_wait();  // s_x and the outputs are ordered after the preceding kernel
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      int n_pair, m_tile;
      tile_coords(pair + i * pairs, n_pair, m_tile);
      const int n_tile = 2 * n_pair + (int)rank;
      const int n = n_tile * kTileN + r;
      const int row_base = m_tile * TW;
      const int t_valid = min(TW, p.M - row_base);
      const float swn = (ystore && n < p.N) ? __ldg(p.s_w + n) : 0.0f;
      // the previous tile's TMA store has read the staging buffer and s_x
      if (et == 0 && ystore) bulk_wait_group_read_all();
      named_bar_sync(1, 128);
      if (ystore)
        for (int j = et; j < TW; j += 128) sx_s[j] = j < t_valid ? p.s_x[row_base + j] : 0.0f;
      // (a wait that runs out raises the CTA's abort flag before the barrier)
      warp_wait(bar_acc + 8 * b, (uint32_t)((i >> 1) & 1), abort_flag, lim);
      tc_fence_after();
      // one thread turns the abort flag into a value every epilogue thread
      // reads between the same two barriers: the branches below (and the
      // barriers inside them) are uniform over the four warps
      named_bar_sync(1, 128);
      if (et == 0) *ep_flag = (*abort_flag == 0 && hdr_ok) ? 1 : 0;
      named_bar_sync(1, 128);
      const bool live = *ep_flag != 0;
      const uint32_t acc_col = (uint32_t)(b * TW);
      if (live) {
        for (int j = 0; j < TW / 16 && 16 * j < t_valid; ++j) {
          uint32_t v[16];
          tmem_ld_x16(lane_base + acc_col + 16 * j, v);
          tmem_wait_ld();
          if (ystore) {
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
          } else if (n < p.N) {
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const int tt = 16 * j + t;
              if (tt < t_valid) p.acc[(size_t)(row_base + tt) * p.N + n] = (int32_t)v[t];
            }
          }
        }
      }
      // the accumulator is free for tile i + 2 (the odd CTA's warps arrive on
      // the even CTA's barrier, after their loads completed)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank != 0)
          mbar_arrive_remote_relaxed(dsmem_map(bar_accfree + 8 * b, 0));
        else
          mbar_arrive(bar_accfree + 8 * b);
      }
      if (live && ystore) {
        fence_proxy_async_smem();  // the staging stores, seen by the TMA engine
        named_bar_sync(1, 128);
        if (et == 0) {
          tma_store_2d(&tmap_y, n_tile * kTileN, row_base, ystage);
          bulk_commit_group();
        }
        __syncwarp();
      }
      if (!live) break;
    }
    if (et == 0 && ystore) bulk_wait_group_all();  // every store performed
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_done);
  }

  // ------------------------------------------------------------ teardown
  if (warp == 1) {
    // every epilogue warp of this CTA is done with tensor memory, and every
    // MMA issued (the even CTA's final commit arrives on both CTAs)
    warp_wait(bar_done, 0, nullptr, kDrainLimitNs);
    warp_wait<true>(bar_fin, 0, nullptr, kDrainLimitNs);
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
  __syncwarp();
  __syncthreads();
  // neither CTA leaves while the other may still arrive on its barriers
  cluster_sync_all();
}

}  // namespace w4a8
