// gemv.cuh -- the W4A8 product for a few tokens (decode, M <= 8) on CUDA
// cores: packed LQQ weights are dequantized to INT8 with the IMAD + XOR
// identity and multiplied with the INT8 activations by 4-way integer dot
// products (dp4a), accumulating exactly in INT32; the same fp32 epilogue as
// the tensor-core kernel then stores bf16 (or the INT32 accumulators).
//
// Method (review page "LiquidGEMM", pith.science verdict on arXiv
// 2509.01229): the dequantization (q_u4 * s_u8 + a) XOR 0x80 per byte, two
// integer instructions per four weights after unpacking (key_machinery;
// referee summary; referee minor 1, paper Sec. 5.3); INT8 x INT8 products
// accumulated in INT32 (lead).  The page's kernel runs the products on
// tensor cores; with one to eight tokens a tensor-core MMA does at most 8 of
// its 128..256 columns of useful work and its issue / commit / TMEM chain is
// the decode critical path, so this form keeps the same arithmetic on the
// CUDA cores, where each dequantized word feeds M dot products directly.
//
// The design (B200):
//   * One CTA (256 threads) owns R output channels (a slice of one 128-row
//     channel block of the packed layout) over a range of at most KR k tiles
//     (128 k each).  One TMA request brings its codes (a 4-D box over the
//     packed tiles: 16 bytes x R rows x 4 chunks x KR tiles) and one its
//     (s_u8, a) pairs (a 3-D box) into shared memory.
//   * The weight copies are issued, and the weights dequantized into
//     registers, before the wait on the preceding kernel (programmatic
//     dependent launch): only the activation copy, the dot products, one
//     reduction and the stores remain on the path after it.
//   * Thread t owns row t % R and P "pieces" (k tile, 32-k chunk) of it;
//     each piece is 8 dequantized words, used for every token.  The S = 256 / R
//     partial sums of a row are added by warp shuffles and one pass through
//     shared memory.
//   * Split-K when K exceeds KR k tiles: the splits of one row slice form a
//     thread-block cluster; every other CTA adds its M x R sums into the
//     leader's shared memory with asynchronous remote adds counted on the
//     leader's mbarrier (no global workspace), and the leader stores.
//   * FUSED: fp32 activations in; the CTA (which then holds the whole row,
//     one split) computes the per-token absmax and quantizes its activations
//     into shared memory with the arithmetic of act_quant_kernel
//     (s = absmax / 127, rint(x / s) clamped to +-127), so the codes and the
//     result equal those of the quantizer followed by the product.
//   * Every wait is bounded; on a timeout the status word records it, no
//     store is made, and the CTA waits (bounded) for its copies in flight.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include "gemm.cuh"
#include "layout.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace w4a8 {

constexpr int kGemvThreads = 256;
constexpr int kGemvMaxM = 8;        // tokens per call
constexpr int kGemvMaxSplits = 8;   // portable cluster size

struct GemvParams {
  const int8_t* Xq;       // [M][K] INT8 activations (not FUSED)
  const float* X;         // [M][K] fp32 activations (FUSED)
  const float* s_x;       // [M] per-token scales (not FUSED, bf16 output)
  const float* s_w;       // packed per-channel scales [n_pad]
  const PackedHeader* hdr;
  uint16_t* Y;            // [M][N] bf16 bits, or nullptr
  int32_t* acc;           // [M][N] int32, or nullptr
  int M, N, K;
  int kt_total;           // K / 128
  int splits, kt_per;     // k tiles per split (<= KR)
  unsigned long long wait_limit_ns;
};

template <int R, int P>
struct GemvCfg {
  static_assert(R == 8 || R == 16, "rows per CTA");
  static constexpr int kS = kGemvThreads / R;   // threads (slots) per row
  static constexpr int kKR = P * kS / 4;        // k tiles per CTA (4 chunks each)
  static_assert(kKR * 4 == P * kS, "pieces cover whole k tiles");
  static_assert(kKR <= 256 && R * 16 <= 256, "TMA box dimensions");
  static constexpr int kWarps = kGemvThreads / 32;
  static constexpr int kCodeBytes = kKR * 4 * R * 16;  // [kt][chunk][row][16 B]
  static constexpr int kPrmBytes = kKR * R * 4;        // [kt][row][(s0, a0, s1, a1)]
  static constexpr int kOffPrm = kCodeBytes;
  static constexpr int kOffRed = (kOffPrm + kPrmBytes + 127) & ~127;  // [warp][m][row] int32
  static constexpr int kRedBytes = kWarps * kGemvMaxM * R * 4;
  static constexpr int kOffRecv = kOffRed + kRedBytes;  // split-K: [m][row] int32
  static constexpr int kRecvBytes = kGemvMaxM * R * 4;
  static constexpr int kOffSx = kOffRecv + kRecvBytes;  // [m] fp32
  static constexpr int kOffAmax = kOffSx + 4 * kGemvMaxM;  // FUSED: [warp][m] fp32
  static constexpr int kOffBar = (kOffAmax + 4 * kWarps * kGemvMaxM + 7) & ~7;
  static constexpr int kOffMisc = kOffBar + 3 * 8;
  static constexpr int kOffX = (kOffMisc + 16 + 127) & ~127;  // [m][KR * 128] int8
  static constexpr int kXRowBytes = kKR * kTileK;
  // dynamic shared memory for M tokens (+ slack to align the base to 128)
  static constexpr int smem_bytes(int M) { return kOffX + M * kXRowBytes + 128; }
};

template <int R, int P, int MINB, bool FUSED>
__global__ void __launch_bounds__(kGemvThreads, MINB)
    w4a8_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes,
                     const __grid_constant__ CUtensorMap tm_prm, const GemvParams p) {
  using C = GemvCfg<R, P>;
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gsm_raw) + 127) & ~uintptr_t(127));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = tid % R, slot = tid / R, chunk = slot & 3;

  const int split = blockIdx.x % p.splits;
  const int n0 = (blockIdx.x / p.splits) * R;   // first channel of the slice
  const int nb = n0 / kTileN, r0 = n0 % kTileN;  // channel block, row within it
  const int kt0 = split * p.kt_per;
  const int nk = min(p.kt_per, p.kt_total - kt0);
  const int M = p.M;
  const uint64_t lim = p.wait_limit_ns;

  const uint32_t bar_w = sbase + C::kOffBar;       // codes + parameters landed
  const uint32_t bar_x = bar_w + 8;                // activations landed
  const uint32_t bar_red = bar_w + 16;             // split-K sums landed (leader)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  volatile int* ep_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int32_t* red = reinterpret_cast<int32_t*>(smem + C::kOffRed);
  int32_t* recv = reinterpret_cast<int32_t*>(smem + C::kOffRecv);
  float* sx_s = reinterpret_cast<float*>(smem + C::kOffSx);
  const int8_t* xs = reinterpret_cast<const int8_t*>(smem + C::kOffX);
  const bool leader = split == 0;

  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_x, 1);
    mbar_init(bar_red, 1);
    *abort_flag = lim == 0 ? 1 : 0;  // a wait budget of 0: abort before any wait
    if (lim == 0) record_status(kDevTimeout);
    fence_barrier_init();
    if (p.splits > 1 && leader)
      mbar_arrive_expect_tx(bar_red, (uint32_t)(p.splits - 1) * (uint32_t)(M * R * 4));
    // the weights do not depend on the preceding kernel: fetch them first
    mbar_arrive_expect_tx(bar_w, (uint32_t)(C::kCodeBytes + C::kPrmBytes));
    tma_load_4d(sbase, &tm_codes, r0 * 16, 0, kt0, nb, bar_w);
    tma_load_3d(sbase + C::kOffPrm, &tm_prm, r0 * 4, kt0, nb, bar_w);
    pdl_launch_dependents();
  }
  if (p.splits > 1 && leader)
    for (int i = tid; i < M * R; i += kGemvThreads) recv[i] = 0;
  __syncthreads();
  if (p.splits > 1) cluster_arrive();  // barriers and the receive buffer exist

  // ---- dequantize this thread's pieces into registers (before the wait on
  // the preceding kernel).  Piece j: k tile kt = slot / 4 + (S / 4) j, chunk
  // `chunk` (k = 32 chunk .. 32 chunk + 31 of that tile); the eight words
  // hold those 32 weights in k order.
  uint32_t d[P][8];
  const bool got_w = mbar_wait(bar_w, 0, abort_flag, lim);
#pragma unroll
  for (int j = 0; j < P; ++j) {
    const int kt = slot / 4 + (C::kS / 4) * j;
    if (got_w && kt < nk) {
      const uint4 v = *reinterpret_cast<const uint4*>(smem + ((kt * 4 + chunk) * R + row) * 16);
      const uint32_t prm = *reinterpret_cast<const uint32_t*>(smem + C::kOffPrm + (kt * R + row) * 4);
      const uint32_t sh = chunk < 2 ? 0 : 16;
      dequant_chunk(v, (prm >> sh) & 0xFFu, ((prm >> (sh + 8)) & 0xFFu) * 0x01010101u, d[j]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) d[j][i] = 0;
    }
  }

  // ---- activations (produced by the preceding kernel)
  pdl_wait();
  const int k_lo = kt0 * kTileK;
  bool hdr_ok = true;
  if (!FUSED) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_x, (uint32_t)(M * nk * kTileK));
      for (int m = 0; m < M; ++m)
        bulk_g2s_plain(sbase + C::kOffX + m * C::kXRowBytes, p.Xq + (size_t)m * p.K + k_lo,
                       (uint32_t)(nk * kTileK), bar_x);
    }
    if (tid < M) sx_s[tid] = p.Y ? p.s_x[tid] : 0.0f;
    if (tid == 32) hdr_ok = p.hdr->magic == kMagic && p.hdr->N == p.N && p.hdr->K == p.K;
    mbar_wait(bar_x, 0, abort_flag, lim);
  } else {
    // per-token absmax over the row (one split: this CTA's range is the row),
    // then the codes of act_quant_kernel written into shared memory
    if (tid == 32) hdr_ok = p.hdr->magic == kMagic && p.hdr->N == p.N && p.hdr->K == p.K;
    float* amax_s = reinterpret_cast<float*>(smem + C::kOffAmax);  // [warp][m]
    const int n4 = nk * (kTileK / 4);
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m) {
      if (m < M) {
        const float4* xr = reinterpret_cast<const float4*>(p.X + (size_t)m * p.K + k_lo);
        float am = 0.0f;
        for (int f = tid; f < n4; f += kGemvThreads) am = fmaxf(am, absmax4(__ldg(xr + f)));
        am = warp_max(am);
        if (lane == 0) amax_s[warp * kGemvMaxM + m] = am;
      }
    }
    __syncthreads();
    if (tid < M) {
      float am = 0.0f;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) am = fmaxf(am, amax_s[w * kGemvMaxM + tid]);
      sx_s[tid] = __fdiv_rn(am, 127.0f);
    }
    __syncthreads();
    uint8_t* xw = smem + C::kOffX;
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m) {
      if (m < M) {
        const float4* xr = reinterpret_cast<const float4*>(p.X + (size_t)m * p.K + k_lo);
        const float s = sx_s[m];
        for (int f = tid; f < n4; f += kGemvThreads)
          *reinterpret_cast<uint32_t*>(xw + m * C::kXRowBytes + 4 * f) = quant4(__ldg(xr + f), s);
      }
    }
  }
  if (tid == 32 && !hdr_ok) record_status(kDevBadPacked);
  if (tid == 32 && !hdr_ok) *abort_flag = 1;  // (no store below)
  __syncthreads();
  const bool live = *abort_flag == 0;

  // ---- dot products: each dequantized word meets the same 4 k of every token
  int acc[kGemvMaxM];
#pragma unroll
  for (int m = 0; m < kGemvMaxM; ++m) acc[m] = 0;
  if (live) {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const int kt = slot / 4 + (C::kS / 4) * j;
      if (kt < nk) {
        const int8_t* xp = xs + kt * kTileK + chunk * 32;
#pragma unroll
        for (int m = 0; m < kGemvMaxM; ++m) {
          if (m < M) {
            const int4 xa = *reinterpret_cast<const int4*>(xp + m * C::kXRowBytes);
            const int4 xb = *reinterpret_cast<const int4*>(xp + m * C::kXRowBytes + 16);
            int a = acc[m];
            a = __dp4a((int)d[j][0], xa.x, a);
            a = __dp4a((int)d[j][1], xa.y, a);
            a = __dp4a((int)d[j][2], xa.z, a);
            a = __dp4a((int)d[j][3], xa.w, a);
            a = __dp4a((int)d[j][4], xb.x, a);
            a = __dp4a((int)d[j][5], xb.y, a);
            a = __dp4a((int)d[j][6], xb.z, a);
            a = __dp4a((int)d[j][7], xb.w, a);
            acc[m] = a;
          }
        }
      }
    }
  }

  // ---- row sums: lanes of one row within a warp, then the warps
#pragma unroll
  for (int m = 0; m < kGemvMaxM; ++m) {
    int v = acc[m];
#pragma unroll
    for (int o = R; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    acc[m] = v;
  }
  if (lane < R) {
#pragma unroll
    for (int m = 0; m < kGemvMaxM; ++m)
      if (m < M) red[(warp * kGemvMaxM + m) * R + row] = acc[m];
  }
  __syncthreads();
  int total = 0;
  const int om = tid / R, orow = tid % R;  // output (token, row) of this thread
  const bool owner = tid < M * R;
  if (owner) {
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) total += red[(w * kGemvMaxM + om) * R + orow];
  }

  // ---- split-K: the other splits add their sums into the leader
  if (p.splits > 1) {
    cluster_wait();
    if (!leader) {
      // every byte the leader expects is sent (zeros after an abort), so its
      // wait ends and it never leaves while adds still land in its memory
      if (owner)
        dsmem_red_async_add_s32(dsmem_map(sbase + C::kOffRecv + 4u * (uint32_t)tid, 0),
                                live ? total : 0, dsmem_map(bar_red, 0));
    } else {
      // (no early exit on this CTA's own abort: the wait covers adds still
      // landing in this CTA's memory)
      if (!mbar_wait<true>(bar_red, 0, nullptr, kDrainLimitNs) && tid == 0) *abort_flag = 1;
      if (owner) total += recv[tid];
    }
  }

  // ---- epilogue: y = bf16(acc * (s_x * s_w)), the tensor-core kernel's rule
  if (tid == 0) *ep_flag = *abort_flag == 0;
  __syncthreads();
  if (owner && leader && *ep_flag) {
    const int n = n0 + orow;
    if (n < p.N) {
      if (p.Y) {
        const float y = (float)total * (sx_s[om] * __ldg(p.s_w + n));
        p.Y[(size_t)om * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      } else {
        p.acc[(size_t)om * p.N + n] = total;
      }
    }
  }
  if (*abort_flag && tid == 0) {
    // let the copies already issued land before the CTA goes away
    mbar_wait(bar_w, 0, nullptr, kDrainLimitNs);
    if (!FUSED) mbar_wait(bar_x, 0, nullptr, kDrainLimitNs);
  }
}

// ---------------------------------------------------------------------------
// The decode form the library uses: the same CTA slice (16 channels x at most
// KR k tiles, loaded by the same two TMA boxes), but the products run as
// warp-level INT8 tensor-core MMAs (mma.sync m16n8k32: 16 channels x 8
// tokens x 32 k per instruction, INT32 accumulators in registers).  The
// dp4a form above turned out issue-bound on this GPU (about 2 us for its
// 64 dot products per thread at one token, measured with per-CTA
// timestamps), while one warp MMA does the work of 32 dp4a for a warp.
//
// Fragments (PTX ISA, mma.m16n8k32 with .s8 operands; g = lane / 4,
// t = lane % 4): A (16 x 32, row-major) a0 = row g, k 4t..4t+3; a1 = row
// g + 8, same k; a2 = row g, k 16 + 4t..; a3 = row g + 8, k 16 + 4t..;
// B (32 x 8) b0 = k 4t..4t+3 of token g, b1 = k 16 + 4t.. of token g;
// D d0, d1 = row g, tokens 2t, 2t + 1; d2, d3 = row g + 8, tokens 2t, 2t + 1.
// In the packed layout, word j of a row's 16-byte chunk holds k 8j..8j+3 in
// its low nibbles and 8j+4..8j+7 in its high nibbles, so the k words t and
// t + 4 of a thread are the low (t even) or high (t odd) nibbles of packed
// words t / 2 and t / 2 + 2: each thread dequantizes exactly the 16 weights
// of its fragment, 4 integer operations per 4 weights.
//
// Warp w takes the chunks q = w + 8 i of the CTA's 4 KR chunks (k tile
// q / 4, chunk q % 4); the eight warps' 16 x 8 partial tiles are added
// through shared memory.  Tokens past M read zeros.
constexpr int kGemvMmaMaxM = 16;  // two groups of 8 tokens (the MMA's N)

template <int KR>
struct GemvMmaCfg {
  static constexpr int kR = 16;
  static constexpr int kMaxM = kGemvMmaMaxM;
  static constexpr int kWarps = kGemvThreads / 32;
  static constexpr int kChunks = 4 * KR;
  static constexpr int kCpw = kChunks / kWarps;  // chunks per warp
  static_assert(kChunks % kWarps == 0, "whole chunks per warp");
  static constexpr int kCodeBytes = KR * 4 * kR * 16;
  static constexpr int kPrmBytes = KR * kR * 4;
  static constexpr int kOffPrm = kCodeBytes;
  // [warp][m][row] int32, rows padded to 17 (fragment stores and the
  // owners' reads both spread over the banks)
  static constexpr int kRedStride = kR + 1;
  static constexpr int kOffRed = (kOffPrm + kPrmBytes + 127) & ~127;
  static constexpr int kRedBytes = kWarps * kMaxM * kRedStride * 4;
  static constexpr int kOffRecv = kOffRed + kRedBytes;  // split-K: [m][row] int32
  static constexpr int kOffSx = kOffRecv + kMaxM * kR * 4;  // [m] fp32
  static constexpr int kOffSw = kOffSx + 4 * kMaxM;           // [row] fp32
  static constexpr int kOffAmax = kOffSw + 4 * kR;            // FUSED: [warp][m] fp32
  static constexpr int kOffBar = (kOffAmax + 4 * kWarps * kMaxM + 7) & ~7;
  static constexpr int kOffMisc = kOffBar + 3 * 8;
  static constexpr int kOffX = (kOffMisc + 16 + 127) & ~127;
  // activation rows padded by 16 bytes: the 8 tokens of a B fragment load
  // fall in different banks
  static constexpr int kXStride = KR * kTileK + 16;
  static constexpr int smem_bytes(int M) { return kOffX + M * kXStride + 128; }
};

__device__ __forceinline__ void mma_s8_16x8x32(int32_t (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four INT8 weights from the low (sh = 0) or high (sh = 4) nibbles of a
// packed word: (code * s + a) XOR 0x80 per byte.
__device__ __forceinline__ uint32_t dequant_word(uint32_t w, uint32_t sh, uint32_t s,
                                                 uint32_t a4) {
  return (((w >> sh) & 0x0F0F0F0Fu) * s + a4) ^ 0x80808080u;
}

// NG: token groups of 8 (1 for M <= 8, 2 for M <= 16); a group's MMAs run
// whatever M is (tokens past M have zero B fragments).
template <int KR, int NG, int MINB, bool FUSED>
__global__ void __launch_bounds__(kGemvThreads, MINB)
    w4a8_gemv_mma_kernel(const __grid_constant__ CUtensorMap tm_codes,
                         const __grid_constant__ CUtensorMap tm_prm, const GemvParams p) {
  using C = GemvMmaCfg<KR>;
  constexpr int R = C::kR;
  extern __shared__ uint8_t gsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(gsm_raw) + 127) & ~uintptr_t(127));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  const int split = blockIdx.x % p.splits;
  const int n0 = (blockIdx.x / p.splits) * R;
  const int nb = n0 / kTileN, r0 = n0 % kTileN;
  const int kt0 = split * p.kt_per;
  const int nk = min(p.kt_per, p.kt_total - kt0);
  const int M = p.M;
  const uint64_t lim = p.wait_limit_ns;

  const uint32_t bar_w = sbase + C::kOffBar;
  const uint32_t bar_x = bar_w + 8;
  const uint32_t bar_red = bar_w + 16;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc);
  int32_t* red = reinterpret_cast<int32_t*>(smem + C::kOffRed);
  int32_t* recv = reinterpret_cast<int32_t*>(smem + C::kOffRecv);
  float* sx_s = reinterpret_cast<float*>(smem + C::kOffSx);
  float* sw_s = reinterpret_cast<float*>(smem + C::kOffSw);
  const bool leader = split == 0;

  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_x, 1);
    mbar_init(bar_red, 1);
    *abort_flag = lim == 0 ? 1 : 0;  // a wait budget of 0: abort before any wait
    if (lim == 0) record_status(kDevTimeout);
    fence_barrier_init();
    if (p.splits > 1 && leader)
      mbar_arrive_expect_tx(bar_red, (uint32_t)(p.splits - 1) * (uint32_t)(M * R * 4));
    // the weights do not depend on the preceding kernel: fetch them first
    mbar_arrive_expect_tx(bar_w, (uint32_t)(C::kCodeBytes + C::kPrmBytes));
    tma_load_4d(sbase, &tm_codes, r0 * 16, 0, kt0, nb, bar_w);
    tma_load_3d(sbase + C::kOffPrm, &tm_prm, r0 * 4, kt0, nb, bar_w);
    pdl_launch_dependents();
  }
  // the epilogue's channel scales (part of the packed weights), early
  if (leader && tid < R) sw_s[tid] = p.Y ? __ldg(p.s_w + n0 + tid) : 0.0f;
  if (p.splits > 1 && leader)
    for (int i = tid; i < M * R; i += kGemvThreads) recv[i] = 0;
  __syncthreads();
  if (p.splits > 1) cluster_arrive();  // barriers and the receive buffer exist

  // ---- this thread's A fragments, dequantized before the wait on the
  // preceding kernel
  uint32_t a[C::kCpw][4];
  const bool got_w = mbar_wait(bar_w, 0, abort_flag, lim);
  {
    const uint32_t sh = (uint32_t)(t & 1) * 4u;
    const int wo = 4 * (t >> 1);  // byte of packed word t / 2 in a row chunk
    // (branch-free: chunks past the k range read the box's other bytes,
    // always inside the shared-memory box, and are zeroed)
#pragma unroll
    for (int i = 0; i < C::kCpw; ++i) {
      const int q = warp + C::kWarps * i, kt = q >> 2, c = q & 3;
      const uint32_t keep = (got_w && kt < nk) ? 0xFFFFFFFFu : 0u;
      const uint8_t* cb = smem + (kt * 4 + c) * R * 16;
      const uint32_t w0 = *reinterpret_cast<const uint32_t*>(cb + g * 16 + wo);
      const uint32_t w1 = *reinterpret_cast<const uint32_t*>(cb + g * 16 + 8 + wo);
      const uint32_t w2 = *reinterpret_cast<const uint32_t*>(cb + (g + 8) * 16 + wo);
      const uint32_t w3 = *reinterpret_cast<const uint32_t*>(cb + (g + 8) * 16 + 8 + wo);
      const uint32_t* pr = reinterpret_cast<const uint32_t*>(smem + C::kOffPrm) + kt * R;
      const uint32_t half = c < 2 ? 0u : 16u;
      const uint32_t pg = pr[g] >> half, ph = pr[g + 8] >> half;
      const uint32_t sg = pg & 0xFFu, ag = ((pg >> 8) & 0xFFu) * 0x01010101u;
      const uint32_t sh8 = ph & 0xFFu, ah = ((ph >> 8) & 0xFFu) * 0x01010101u;
      a[i][0] = dequant_word(w0, sh, sg, ag) & keep;
      a[i][1] = dequant_word(w2, sh, sh8, ah) & keep;
      a[i][2] = dequant_word(w1, sh, sg, ag) & keep;
      a[i][3] = dequant_word(w3, sh, sh8, ah) & keep;
    }
  }

  // ---- activations (produced by the preceding kernel)
  pdl_wait();
  const int k_lo = kt0 * kTileK;
  bool hdr_ok = true;
  if (!FUSED) {
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_x, (uint32_t)(M * nk * kTileK));
      for (int m = 0; m < M; ++m)
        bulk_g2s_plain(sbase + C::kOffX + m * C::kXStride, p.Xq + (size_t)m * p.K + k_lo,
                       (uint32_t)(nk * kTileK), bar_x);
    }
    if (tid < M) sx_s[tid] = p.Y ? p.s_x[tid] : 0.0f;
    if (tid == 32) hdr_ok = p.hdr->magic == kMagic && p.hdr->N == p.N && p.hdr->K == p.K;
    mbar_wait(bar_x, 0, abort_flag, lim);
  } else {
    // per-token absmax over the row (one split: this CTA's range is the row),
    // then the codes of act_quant_kernel written into shared memory
    if (tid == 32) hdr_ok = p.hdr->magic == kMagic && p.hdr->N == p.N && p.hdr->K == p.K;
    float* amax_s = reinterpret_cast<float*>(smem + C::kOffAmax);  // [warp][m]
    const int n4 = nk * (kTileK / 4);
    // float4 f = tid + 256 j of a token row (at most kF4 per thread): every
    // load of a token is issued before any is used (one L2 round trip, not
    // one per float4)
    constexpr int kF4 = KR * (kTileK / 4) / kGemvThreads;
#pragma unroll
    for (int m = 0; m < 8 * NG; ++m) {
      if (m < M) {
        const float4* xr = reinterpret_cast<const float4*>(p.X + (size_t)m * p.K + k_lo);
        float4 v[kF4];
#pragma unroll
        for (int j = 0; j < kF4; ++j) {
          const int f = tid + kGemvThreads * j;
          v[j] = f < n4 ? __ldg(xr + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float am = 0.0f;
#pragma unroll
        for (int j = 0; j < kF4; ++j) am = fmaxf(am, absmax4(v[j]));
        am = warp_max(am);
        if (lane == 0) amax_s[warp * C::kMaxM + m] = am;
      }
    }
    __syncthreads();
    if (tid < M) {
      float am = 0.0f;
#pragma unroll
      for (int w = 0; w < C::kWarps; ++w) am = fmaxf(am, amax_s[w * C::kMaxM + tid]);
      sx_s[tid] = __fdiv_rn(am, 127.0f);
    }
    __syncthreads();
    uint8_t* xw = smem + C::kOffX;
#pragma unroll
    for (int m = 0; m < 8 * NG; ++m) {
      if (m < M) {
        const float4* xr = reinterpret_cast<const float4*>(p.X + (size_t)m * p.K + k_lo);
        const float s = sx_s[m];
        uint8_t* xm = xw + m * C::kXStride;
        // (the row is read again: an L1 hit)
        float4 v[kF4];
#pragma unroll
        for (int j = 0; j < kF4; ++j) {
          const int f = tid + kGemvThreads * j;
          v[j] = f < n4 ? __ldg(xr + f) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (rcp_quant_ok(s)) {  // (uniform: one scale per token)
          const float y = __fdiv_rn(1.0f, s);
#pragma unroll
          for (int j = 0; j < kF4; ++j) {
            const int f = tid + kGemvThreads * j;
            if (f < n4) *reinterpret_cast<uint32_t*>(xm + 4 * f) = quant4_rcp(v[j], s, y);
          }
        } else {
#pragma unroll
          for (int j = 0; j < kF4; ++j) {
            const int f = tid + kGemvThreads * j;
            if (f < n4) *reinterpret_cast<uint32_t*>(xm + 4 * f) = quant4(v[j], s);
          }
        }
      }
    }
  }
  if (tid == 32 && !hdr_ok) {
    record_status(kDevBadPacked);
    *abort_flag = 1;  // (no store below)
  }
  __syncthreads();
  const bool live = *abort_flag == 0;

  // ---- warp MMAs.  Every MMA is issued unconditionally: chunks past this
  // CTA's k range and tokens past M have zero B fragments (the A fragments
  // of those chunks are zero too).  A runtime branch around the
  // warp-collective mma.sync, uniform or not, measured about 140 cycles per
  // chunk on this GPU (the loop took 2900 cycles instead of 670).  All B
  // fragments are read with select, not under a branch; two accumulator
  // sets halve the MMA chain.
  // accumulator chains: two per group of one (independent chains halve the
  // MMA latency chain), one per group of two (the groups interleave)
  constexpr int ND = NG == 1 ? 2 : NG;
  int32_t d[ND][4];
#pragma unroll
  for (int j = 0; j < ND; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0;
  if (live) {
    const uint8_t* xg[NG];
    bool tok[NG];
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      const int tk = 8 * gr + g;  // this lane's token in group gr
      tok[gr] = tk < M;
      xg[gr] = smem + C::kOffX + (tok[gr] ? tk : 0) * C::kXStride + 4 * t;
    }
#pragma unroll
    for (int i = 0; i < C::kCpw; ++i) {
      const int q = warp + C::kWarps * i, kt = q >> 2, c = q & 3;
#pragma unroll
      for (int gr = 0; gr < NG; ++gr) {
        const bool use = tok[gr] && kt < nk;
        const uint8_t* xp = xg[gr] + kt * kTileK + c * 32;  // inside the buffer for kt < KR
        const uint32_t b0 = use ? *reinterpret_cast<const uint32_t*>(xp) : 0u;
        const uint32_t b1 = use ? *reinterpret_cast<const uint32_t*>(xp + 16) : 0u;
        mma_s8_16x8x32(d[NG == 1 ? (i & 1) : gr], a[i], b0, b1);
      }
    }
  }
  // the warps' partial tiles: red[warp][token][row]
  constexpr int RS = C::kRedStride;
#pragma unroll
  for (int gr = 0; gr < NG; ++gr) {
    const int32_t* dd = d[NG == 1 ? 0 : gr];
    const int32_t* de = NG == 1 ? d[1] : nullptr;
    int32_t* rw = red + (warp * C::kMaxM + 8 * gr) * RS;
    rw[(2 * t) * RS + g] = dd[0] + (de ? de[0] : 0);
    rw[(2 * t + 1) * RS + g] = dd[1] + (de ? de[1] : 0);
    rw[(2 * t) * RS + g + 8] = dd[2] + (de ? de[2] : 0);
    rw[(2 * t + 1) * RS + g + 8] = dd[3] + (de ? de[3] : 0);
  }
  __syncthreads();
  int total = 0;
  const int om = tid / R, orow = tid % R;  // output (token, row) of this thread
  const bool owner = tid < M * R;
  if (owner) {
#pragma unroll
    for (int w = 0; w < C::kWarps; ++w) total += red[(w * C::kMaxM + om) * RS + orow];
  }

  // ---- split-K: the other splits add their sums into the leader
  if (p.splits > 1) {
    cluster_wait();
    if (!leader) {
      // every byte the leader expects is sent (zeros after an abort), so its
      // wait ends and it never leaves while adds still land in its memory
      if (owner)
        dsmem_red_async_add_s32(dsmem_map(sbase + C::kOffRecv + 4u * (uint32_t)tid, 0),
                                live ? total : 0, dsmem_map(bar_red, 0));
    } else {
      // (no early exit on this CTA's own abort: the wait covers adds still
      // landing in this CTA's memory)
      if (!mbar_wait<true>(bar_red, 0, nullptr, kDrainLimitNs) && tid == 0) *abort_flag = 1;
      if (owner) total += recv[tid];
    }
  }

  // ---- epilogue: y = bf16(acc * (s_x * s_w)), the tensor-core kernel's rule
  if (p.splits > 1 && leader) __syncthreads();  // abort raised by the wait above
  if (owner && leader && *abort_flag == 0) {
    const int n = n0 + orow;
    if (n < p.N) {
      if (p.Y) {
        const float y = (float)total * (sx_s[om] * sw_s[orow]);
        p.Y[(size_t)om * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
      } else {
        p.acc[(size_t)om * p.N + n] = total;
      }
    }
  }
  if (*abort_flag && tid == 0) {
    // let the copies already issued land before the CTA goes away
    mbar_wait(bar_w, 0, nullptr, kDrainLimitNs);
    if (!FUSED) mbar_wait(bar_x, 0, nullptr, kDrainLimitNs);
  }
}

}  // namespace w4a8
