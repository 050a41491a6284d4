/*
 * w4a8.h -- C ABI of libw4a8.so, a block-quantized W4A8 GEMM for NVIDIA
 * B200 (sm_100a) in the style of LiquidGEMM / LiquidQuant (LQQ).
 *
 * The method (review page "LiquidGEMM", pith.science verdict on arXiv
 * 2509.01229; field names of that page and the paper sections they quote):
 *   - weights: per-output-channel symmetric INT8 in the protective range
 *     [-119, 119] with an FP scale s_w (referee major 3, paper Sec. 4 Eq. 7),
 *     then per group of 64 along K (skeptic concrete_test) shifted by the
 *     group minimum into UINT8 and quantized to UINT4 codes with an integer
 *     scale s_u8 <= 16 and an offset a = 2^7 + min (referee summary;
 *     key_machinery; referee minor 2, Sec. 4 Eq. 10);
 *   - dequantization inside the GEMM: (q_u4 * s_u8 + a) XOR 0x80, integer
 *     multiply-add and a bit flip that never leave UINT8 (key_machinery;
 *     referee summary; desk_editor);
 *   - activations: per-token INT8 with an FP scale (supporting citation [29]);
 *   - INT8 x INT8 tensor-core products accumulated in INT32 (lead), followed
 *     by an FP epilogue y = s_x[m] * s_w[n] * acc[m][n] stored as bf16.
 *
 * Conventions for every entry point:
 *   - Pointers named X, W, Xq, s_x, packed, Y, acc and the outputs
 *     of the unpack call are DEVICE pointers owned by the caller.  The library
 *     allocates no memory and never synchronizes the host, except in
 *     w4a8_get_status.  Work is enqueued on `stream` (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream) in call order.
 *   - Matrices are row-major with the last index contiguous:
 *       W  float32 [N][K]  (output channel n, reduction index k)
 *       X  float32 [M][K]  (token m)
 *       Xq int8    [M][K],  s_x float32 [M]
 *       Y  bf16    [M][N]   (stored as uint16 bit patterns)
 *       acc int32  [M][N]
 *   - Supported shapes: M >= 0, N >= 1, K a positive multiple of 128,
 *     K <= 65536, group = 64 or 128.  M == 0 is a no-op.  Other shapes return
 *     W4A8_ERR_UNSUPPORTED_SHAPE before anything is launched.
 *   - Alignment: Xq, X, W and the packed buffer must be 16-byte aligned,
 *     acc and every float32 scale array 4-byte aligned, Y 2-byte aligned;
 *     otherwise W4A8_ERR_MISALIGNED.  Y only needs its element alignment;
 *     a more aligned Y enables faster stores: 16-byte alignment with N a
 *     multiple of 8 lets dense calls without split-K write whole tiles with
 *     a TMA tensor store, 8-byte alignment with N a multiple of 4 lets
 *     split-K reductions store four channels per instruction.
 *   - Return value: W4A8_OK or a negative w4a8_status.  Argument errors are
 *     detected on the host before any launch.  A launch failure returns
 *     W4A8_ERR_CUDA.  Errors found on the device (a bounded wait that ran out)
 *     are recorded in a per-device status word read by w4a8_get_status.
 *   - Inputs must be finite; NaN or Inf inputs give unspecified codes.
 */
#ifndef W4A8_H
#define W4A8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4A8_OK = 0,
  W4A8_ERR_INVALID_ARG = -1,       /* NULL pointer, negative size, bad group */
  W4A8_ERR_UNSUPPORTED_SHAPE = -2, /* K % 128, K > 65536, N < 1 */
  W4A8_ERR_MISALIGNED = -3,        /* see the alignment rule above */
  W4A8_ERR_CUDA = -5,              /* a CUDA runtime call failed */
  W4A8_ERR_TIMEOUT = -6,           /* a device-side bounded wait ran out */
  W4A8_ERR_BAD_PACKED = -7,        /* packed buffer header does not match */
  W4A8_ERR_BAD_OFFSETS = -8        /* grouped GEMM: invalid row offsets */
} w4a8_status;

/* Human-readable name of a status code.  Never NULL. */
const char* w4a8_status_string(int status);

/* Library ABI version (currently 1). */
int w4a8_version(void);

/*
 * Size in bytes of the packed LQQ weight buffer for an N x K layer.
 * Layout (all offsets from the buffer start):
 *   [0, 256)       header: magic 'W4A8', version, N, K, group, padded N
 *   [256, ...)     s_w: float32 per output channel, N rounded up to 128
 *   tiles          one 8704-byte tile per (128 output channels, 128 k):
 *                  8192 bytes of 4-bit codes then 512 bytes of (s_u8, a)
 *                  pairs, tiles ordered by output-channel block, then k.
 * Returns 0 for an unsupported shape.  Host-only, no CUDA call.
 */
size_t w4a8_packed_weight_bytes(int N, int K, int group);

/*
 * Offline weight quantization and packing (review: key_machinery; referee
 * summary; referee major 3 and minor 2, paper Sec. 4 Eqs. 7 and 10).
 *   W       [N][K] float32, device
 *   packed  device buffer of w4a8_packed_weight_bytes(N, K, group) bytes,
 *           every byte written by this call (header tail and padding
 *           channels included), so the buffer can be saved and reloaded
 * Level 1: s_w[n] = max_k |W[n][k]| / 119 (fp32 division);
 *          Q = clamp(rint(W / s_w), -119, 119), ties to even; s_w = 0 gives 0.
 * Level 2, per group of `group` k-values in one row: mn/mx = min/max of Q,
 *          s_u8 = max(1, ceil((mx - mn) / 15)), a = 128 + mn,
 *          code = floor((2 (Q - mn) + s_u8) / (2 s_u8)) in [0, 15].
 */
int w4a8_quantize_weights(const float* W, int N, int K, int group,
                          void* packed, void* stream);

/*
 * Test aid: expand a packed buffer back into canonical arrays.
 *   codes [N][K] uint8 (one code per byte), s_u8 [N][K/group] uint8,
 *   a [N][K/group] uint8, s_w [N] float32.  All device pointers.
 * N, K and group are read from the header; pass the same N and K as a check.
 */
int w4a8_unpack_weights(const void* packed, int N, int K, uint8_t* codes,
                        uint8_t* s_u8, uint8_t* a, float* s_w, void* stream);

/*
 * Per-token activation quantization (supporting citation [29]; symmetric
 * range +-127):  s_x[m] = max_k |X[m][k]| / 127 (fp32 division),
 * Xq[m][k] = clamp(rint(X[m][k] / s_x[m]), -127, 127), ties to even;
 * an all-zero row gives s_x = 0 and Xq = 0.
 *   X [M][K] float32 -> Xq [M][K] int8, s_x [M] float32 (device).
 * K only needs to be a positive multiple of 16 here.
 */
int w4a8_quantize_act(const float* X, int M, int K, int8_t* Xq, float* s_x,
                      void* stream);

/*
 * The W4A8 GEMM with the fused bf16 epilogue:
 *   Y[m][n] = bf16_rn( float(acc[m][n]) * (s_x[m] * s_w[n]) ),
 *   acc[m][n] = sum_k Xq[m][k] * (code[n][k] * s_u8 + a - 128)   (INT32)
 * with the weights dequantized in-kernel as (code * s_u8 + a) XOR 0x80
 * (key_machinery) and the products on tcgen05 INT8 tensor cores (lead).
 *   Xq [M][K] int8, s_x [M] float32, packed (from w4a8_quantize_weights;
 *   the caller must pass the N and K it was built for), Y [M][N] bf16.
 * The accumulator is exact; the epilogue differs from an exact FP64
 * evaluation by at most one bf16 ulp.  Shapes with few output tiles split K
 * across a thread-block cluster of up to 8 CTAs whose partial sums are
 * reduced on chip, so no scratch memory is needed.
 */
int w4a8_gemm(const int8_t* Xq, const float* s_x, const void* packed, int M,
              int N, int K, uint16_t* Y, void* stream);

/*
 * Launch options for the *_ex entry points (bit mask).
 * W4A8_FLAG_PDL: launch with programmatic dependent launch.  The kernel may
 *   start while the kernel before it in the stream is still running; it
 *   waits for that kernel's results before reading its activation inputs or
 *   writing anything, but it reads the packed weights (and their scales)
 *   early.  Use it only when the preceding kernel in the stream does not
 *   write the packed weight buffer.  This hides launch and weight-fetch
 *   latency in chains of small calls (decode).
 */
#define W4A8_FLAG_PDL 1u

/*
 * W4A8_FLAG_TENSOR_CORE (w4a8_gemm_ex, w4a8_gemm_fused): run the
 *   tcgen05 kernel even where the library would take the decode form for a
 *   few tokens (w4a8_gemm_kernel_kind).  The result is
 *   bit-identical either way; the flag exists to compare and test the two.
 */
#define W4A8_FLAG_TENSOR_CORE 2u

/* w4a8_gemm with launch options (flags as above; 0 = w4a8_gemm). */
int w4a8_gemm_ex(const int8_t* Xq, const float* s_x, const void* packed, int M,
                 int N, int K, uint16_t* Y, unsigned flags, void* stream);

/* w4a8_quantize_act with launch options (flags as above).  With
 * W4A8_FLAG_PDL it waits for the preceding kernel before reading X. */
int w4a8_quantize_act_ex(const float* X, int M, int K, int8_t* Xq, float* s_x,
                         unsigned flags, void* stream);

/* Same product, writing the exact INT32 accumulators acc [M][N] instead of
 * the bf16 output (for bit-exact verification). */
int w4a8_gemm_i32(const int8_t* Xq, const void* packed, int M, int N, int K,
                  int32_t* acc, void* stream);

/*
 * Schedule the library picks for a shape (introspection for tests and
 * benchmarks): tokens per tile, split-K factor (= cluster size), number of
 * CTAs.  Any output
 * pointer may be NULL.  Host-only.
 */
int w4a8_gemm_schedule(int M, int N, int K, int* tile_tokens, int* splits,
                       int* ctas);

/*
 * Which kernel w4a8_gemm / w4a8_gemm_i32 run for a shape (host-only):
 *   W4A8_KERNEL_TENSOR_CORE  tcgen05 INT8 MMAs, weights dequantized into
 *                            tensor memory (lead; key_machinery)
 *   W4A8_KERNEL_WARP_MMA     the decode form for a few tokens: the same
 *                            IMAD + XOR dequantization (key_machinery) into
 *                            registers and warp-level INT8 tensor-core MMAs
 *                            (mma.sync) with INT32 accumulators, 16 output
 *                            channels per CTA; w4a8_gemm_schedule then
 *                            reports tile_tokens = M
 * Both give bit-identical results.  Negative status for a bad shape.
 */
#define W4A8_KERNEL_TENSOR_CORE 0
#define W4A8_KERNEL_WARP_MMA 1
int w4a8_gemm_kernel_kind(int M, int N, int K);

/*
 * ---- Activation quantization fused into the GEMM (decode) ----
 * The same product as w4a8_quantize_act followed by w4a8_gemm, in one
 * launch (the per-token quantizer of supporting citation [29] moved into the
 * GEMM's producer): the GEMM's producer and MMA warps read the fp32
 * activations of their k range into registers, combine the per-token absmax
 * across the split-K cluster, and quantize straight into the MMA's operand
 * tiles.  The rule and its arithmetic are w4a8_quantize_act's (s_x =
 * absmax / 127, codes rint(x / s_x) clamped to +-127), so Y is bit-identical
 * to the two-call form.
 *   X [M][K] float32 (16-byte aligned), packed as for w4a8_gemm, Y [M][N]
 *   bf16; all device pointers.  flags: W4A8_FLAG_PDL or 0.
 * Applies to decode shapes only (w4a8_gemm_fused_supported): M <= 16 with
 * the 16-token tile, at most 6 k tiles per CTA, M x (k tiles per CTA) <= 16
 * (the CTA's slice of X fits the two warps' registers), and split-K only for
 * M <= 8.  Other shapes return W4A8_ERR_UNSUPPORTED_SHAPE before any launch.
 * On B200 the two calls chained with W4A8_FLAG_PDL are faster (4096 x 4096,
 * M = 1: about 6.3 us per pair against 8.6 us): the fused kernel puts the
 * activation reads, the cluster exchange and the quantization in front of
 * its first MMA, where the pair overlaps the quantizer with the GEMM's weight
 * prefetch and dequantization.
 */
int w4a8_gemm_fused(const float* X, const void* packed, int M, int N, int K,
                    uint16_t* Y, unsigned flags, void* stream);

/* 1 if w4a8_gemm_fused applies to the shape on the current device, else 0.
 * Host-only. */
int w4a8_gemm_fused_supported(int M, int N, int K);

/*
 * ---- Ablation variants ----
 * The review page reports an ablation of the method's parts (referee
 * significance: LQQ, ImFP and their effect on throughput).  These variants
 * each change one design decision of this library's kernel against a fixed
 * baseline, and compute exactly the same result:
 *   BASELINE          16-token tile with the deep ring (10 stages) for
 *                     M <= 16, else the 256-token tile; two dequantization
 *                     warpgroups, a dedicated MMA warp, 4 TMEM weight
 *                     slots, gather split-K reduction, the library's splits
 *   NAIVE_DEQUANT     each 4-bit code unpacked on its own, code * s + min in
 *                     signed 32-bit arithmetic, saturated to INT8 and packed
 *                     (instead of two instructions per four weights)
 *   ONE_GROUP         one dequantization warpgroup instead of two
 *   SERIAL            one dequantization warpgroup and one TMEM weight slot:
 *                     dequantizing a k tile waits for the MMAs of the
 *                     previous one (no overlap of the two)
 *   GROUP_ISSUES_MMA  one dequantization warpgroup that also issues the MMAs
 *                     (no dedicated MMA warp)
 *   CTA_PAIR          the 256-token tile computed by a pair of CTAs with
 *                     CTA-pair MMAs (tcgen05 cta_group::2): each CTA holds
 *                     its 128 channels and loads half of the tokens, with an
 *                     8-deep ring; no split-K.  Needs M >= 256 and an even
 *                     number of 128-channel blocks (else
 *                     W4A8_ERR_UNSUPPORTED_SHAPE).  The default uses this
 *                     form wherever it applies.
 *   TENSOR_CORE       the tcgen05 kernel in the library's schedule for
 *                     every M (the default takes the decode form below for
 *                     a few tokens)
 *   WARP_MMA          the decode form (w4a8_gemm_kernel_kind): 16 output
 *                     channels per CTA, weights dequantized into registers,
 *                     warp-level INT8 MMAs (mma.sync m16n8k32); 1 <= M <= 8,
 *                     K <= 32768 (else W4A8_ERR_UNSUPPORTED_SHAPE)
 *   DP4A              the decode form with CUDA-core 4-way dot products
 *                     (dp4a) instead of warp MMAs; same limits
 *   PERSISTENT        the persistent CTA-pair form for any M: one CTA pair
 *                     per two SMs walks 256-channel x 192-token output
 *                     tiles; two accumulators in tensor memory, so a tile's
 *                     epilogue (dedicated warps, one TMA store per tile)
 *                     overlaps the next tile's main loop.  Needs an even
 *                     number of 128-channel blocks and, for bf16 output, N a
 *                     multiple of 8 and Y 16-byte aligned (else
 *                     W4A8_ERR_UNSUPPORTED_SHAPE).  An ablation: measured
 *                     no faster than CTA_PAIR, so the default never takes it.
 * DEFAULT is the library's own choice (w4a8_gemm_ex / w4a8_gemm_i32).
 * Exactly one of Y (bf16, with s_x) or acc (INT32) is non-NULL.  Other
 * arguments as for w4a8_gemm_ex.
 */
#define W4A8_VARIANT_DEFAULT 0
#define W4A8_VARIANT_BASELINE 1
#define W4A8_VARIANT_NAIVE_DEQUANT 2
#define W4A8_VARIANT_SERIAL 3
#define W4A8_VARIANT_ONE_GROUP 4
#define W4A8_VARIANT_GROUP_ISSUES_MMA 5
#define W4A8_VARIANT_CTA_PAIR 6
#define W4A8_VARIANT_TENSOR_CORE 7
#define W4A8_VARIANT_DP4A 8
#define W4A8_VARIANT_WARP_MMA 9
#define W4A8_VARIANT_PERSISTENT 10

int w4a8_gemm_variant(int variant, const int8_t* Xq, const float* s_x,
                      const void* packed, int M, int N, int K, uint16_t* Y,
                      int32_t* acc, unsigned flags, void* stream);

/*
 * ---- Grouped GEMM for mixture-of-experts layers ----
 * The pages serve Mixtral-8x7B (skeptic's concrete test), whose expert
 * layers are many W4A8 GEMMs of one shape with a variable number of tokens
 * each.  One launch covers all of them:
 *   for every group g and row m in [offsets[g], offsets[g+1]):
 *     Y[m][n] = bf16_rn( float(acc) * (s_x[m] * s_w_g[n]) ),
 *     acc = sum_k Xq[m][k] * Wdq_g[n][k]
 * with the rows of Xq / Y grouped by expert (the caller sorts tokens by
 * expert; a token routed to two experts appears twice).
 *   packed:  `groups` packed buffers of one (N, K, group), back to back,
 *            w4a8_packed_weight_bytes(N, K, group) bytes apart (group g's
 *            buffer starts g times that many bytes after `packed`).
 *   offsets: int32 [groups + 1] on the DEVICE: offsets[0] = 0, nondecreasing,
 *            offsets[groups] = M_total.  It may be written by the preceding
 *            kernel in the stream (with W4A8_FLAG_PDL the kernel waits for it).
 *   max_rows: host-side bound on the rows of any one group (1..M_total);
 *            it sizes the launch and the tile width, so a tight bound is
 *            faster.  Xq [M_total][K], s_x [M_total], Y [M_total][N].
 * If any group's offsets are out of order, outside [0, M_total] or span
 * more than max_rows rows, the call stores nothing and w4a8_get_status
 * reports W4A8_ERR_BAD_OFFSETS.  The launch has one CTA per token tile that
 * can hold rows (at most ceil(M_total / T) + groups - 1 of them, T the tile
 * width) times the channel blocks and splits, so empty experts cost nothing.
 */
int w4a8_grouped_gemm(const int8_t* Xq, const float* s_x, const void* packed,
                      int groups, const int* offsets, int M_total, int max_rows,
                      int N, int K, uint16_t* Y, unsigned flags, void* stream);

/* The grouped product's exact INT32 accumulators acc [M_total][N]. */
int w4a8_grouped_gemm_i32(const int8_t* Xq, const void* packed, int groups,
                          const int* offsets, int M_total, int max_rows, int N,
                          int K, int32_t* acc, void* stream);

/* Schedule of the grouped kernel (as w4a8_gemm_schedule; ctas counts the
 * CTAs launched, including token-tile slots that find no rows and exit). */
int w4a8_grouped_gemm_schedule(int groups, int M_total, int max_rows, int N,
                               int K, int* tile_tokens, int* splits, int* ctas);

/*
 * ---- W8A8 comparison point ----
 * The review page (pith summary; forward implication 3) measures the method
 * against W8A8: 8-bit weights that need no dequantization.  These entry
 * points run that product on the same kernel, rings, split-K reduction and
 * epilogue, so that the two weight formats can be compared on one harness.
 *
 * Per-channel symmetric INT8 weights, by the same rule as the activations:
 *   s_w[n] = max_k |W[n][k]| / 127 (fp32 division),
 *   Wq[n][k] = clamp(rint(W[n][k] / s_w[n]), -127, 127), ties to even;
 *   an all-zero channel gives s_w = 0 and Wq = 0.
 *   W [N][K] float32 -> Wq [N][K] int8 (row-major, 16-byte aligned),
 *   s_w [N] float32 (device, caller-owned).  K must be a multiple of 128.
 */
int w8a8_quantize_weights(const float* W, int N, int K, int8_t* Wq, float* s_w,
                          void* stream);

/*
 * Y[m][n] = bf16_rn( float(acc[m][n]) * (s_x[m] * s_w[n]) ),
 * acc[m][n] = sum_k Xq[m][k] * Wq[n][k]   (INT32, exact).
 *   Xq [M][K] int8, s_x [M] float32, Wq [N][K] int8, s_w [N] float32,
 *   Y [M][N] bf16 (all device, caller-owned; Xq and Wq 16-byte aligned).
 * flags: W4A8_FLAG_PDL or 0.  Same shape rules and error codes as w4a8_gemm.
 */
int w8a8_gemm(const int8_t* Xq, const float* s_x, const int8_t* Wq,
              const float* s_w, int M, int N, int K, uint16_t* Y,
              unsigned flags, void* stream);

/* The W8A8 product's exact INT32 accumulators acc [M][N]. */
int w8a8_gemm_i32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                  int32_t* acc, void* stream);

/* Schedule of the W8A8 kernel for a shape (as w4a8_gemm_schedule). */
int w8a8_gemm_schedule(int M, int N, int K, int* tile_tokens, int* splits,
                       int* ctas);

/*
 * Waits for `stream`, then returns and clears the device status word of the
 * current device: W4A8_OK, or W4A8_ERR_TIMEOUT if a kernel's bounded wait
 * ran out since the last call.  W4A8_ERR_CUDA if the synchronization failed.
 */
int w4a8_get_status(void* stream);

/*
 * Test aid for the failure path: launches one CTA that waits on a shared
 * memory barrier nothing ever arrives on, with a wait limit of `limit_ns`
 * nanoseconds (1e3 .. 1e10).  The kernel records W4A8_ERR_TIMEOUT in the
 * status word and returns; nothing faults or hangs.
 */
int w4a8_debug_timeout_probe(long long limit_ns, void* stream);

/*
 * Test aid for the GEMM's own failure path: the budget, in nanoseconds, of
 * the main-loop waits of every kernel launched afterwards by this process
 * (all entry points, all devices).  -1 restores the default of 2 s; 0 makes
 * every CTA of each launch raise its abort flag at set-up, before any wait,
 * so each of those waits that does not find its phase complete gives up at
 * once and the launch runs its abort path: the
 * status word records W4A8_ERR_TIMEOUT, nothing is stored, and the kernel
 * first waits (always with the full 2 s budget) for the copies, MMAs and
 * remote adds it already started, then frees its tensor memory and returns.
 * Valid range -1 .. 1e10; otherwise W4A8_ERR_INVALID_ARG.  Host-only; the
 * setting is read when a call launches its kernel.
 */
int w4a8_debug_set_wait_budget(long long ns);

#ifdef __cplusplus
}
#endif

#endif /* W4A8_H */
