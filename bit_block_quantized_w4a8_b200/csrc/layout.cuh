// layout.cuh -- the packed LQQ weight layout consumed by the GEMM kernel.
//
// The packed buffer is built once per layer (offline) so that one 1-D bulk
// copy moves everything the kernel needs for 128 output channels x 128 k
// into shared memory, and so that each dequantization thread (one per output
// channel = one TMEM lane) reads its 16-byte code chunks without shared
// memory bank conflicts.
//
//   header  [0, 256): PackedHeader
//   s_w     [256, 256 + 4*Np): float32 per output channel (Np = N rounded up
//           to 128; padding channels have s_w = 0)
//   tiles   from tiles_offset: (Np/128) x (K/128) tiles of kTileBytes,
//           ordered by channel block nb, then k block kb.
//
// One tile (channel block nb, k block kb), rows r = 0..127 are the channels
// n = 128 nb + r and k runs over 128 kb .. 128 kb + 127:
//   codes   [0, 8192): chunk c (k = 32c .. 32c + 31 of the tile), row r at
//           byte offset (c * 128 + r) * 16.  The 16 bytes are four 32-bit
//           words; word j holds k = 32c + 8j .. 32c + 8j + 7: byte b of the
//           word has the code of k = 32c + 8j + b in its low nibble and the
//           code of k = 32c + 8j + 4 + b in its high nibble.  So
//           w & 0x0F0F0F0F and (w >> 4) & 0x0F0F0F0F are two words of four
//           codes each, in k order.
//   params  [8192, 8704): row r at byte offset 8192 + 4 r holds
//           (s_u8, a) of the group covering tile k 0..63, then (s_u8, a) of
//           the group covering tile k 64..127 (for group 128 both are equal).
// Padding channels (n >= N) have codes 0, s_u8 = 1 and a = 128, which
// dequantize to 0.
#pragma once
#include <cstddef>
#include <cstdint>

namespace w4a8 {

constexpr int kTileN = 128;                 // output channels per tile
constexpr int kTileK = 128;                 // k values per tile
constexpr int kCodeBytes = kTileN * kTileK / 2;   // 8192
constexpr int kParamBytes = kTileN * 4;           // 512
constexpr int kTileBytes = kCodeBytes + kParamBytes;  // 8704
constexpr int kHeaderBytes = 256;
constexpr uint32_t kMagic = 0x38413457u;    // "W4A8" little-endian
constexpr uint32_t kLayoutVersion = 1;

struct PackedHeader {
  uint32_t magic;
  uint32_t version;
  int32_t N;
  int32_t K;
  int32_t group;
  int32_t n_pad;
  uint64_t sw_offset;
  uint64_t tiles_offset;
  uint64_t total_bytes;
};
static_assert(sizeof(PackedHeader) == 48 && sizeof(PackedHeader) <= kHeaderBytes,
              "packed header fields");

__host__ __device__ inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

__host__ __device__ inline uint64_t sw_offset_bytes() { return kHeaderBytes; }

__host__ __device__ inline uint64_t tiles_offset_bytes(int n_pad) {
  uint64_t end = kHeaderBytes + 4ull * (uint64_t)n_pad;
  return (end + 255) / 256 * 256;
}

__host__ __device__ inline uint64_t packed_bytes(int N, int K) {
  int np = round_up(N, kTileN);
  return tiles_offset_bytes(np) +
         (uint64_t)(np / kTileN) * (uint64_t)(K / kTileK) * kTileBytes;
}

}  // namespace w4a8
