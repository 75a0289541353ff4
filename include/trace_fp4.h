/*
 * trace_fp4.h -- C ABI of the block-scaled FP4 quantization library for
 * rollout-guided FP4 quantization-aware training, NVIDIA B200 (sm_100a).
 *
 * Method (web pages, cited by title and section):
 *   - "TRACE: Rollout-Guided Quantization-Aware Training for FP4
 *     Reinforcement Learning of MoE Language Models", summary at
 *     ai-papers.net: sections "学習とロールアウトの不一致" (nearest rounding
 *     sends nearby values to different codewords), "TRACEの仕組み" (the
 *     train side rounds each value to whichever of its two adjacent
 *     codewords the rollout chose; straight-through backward) and
 *     "量子化情報キャッシュ" (keep only the mantissa bit and the scale, only
 *     for the deeper layers -- about 1/6 of the full information).
 *   - Korean explainer of the same paper (sns.style), "작동 원리": the
 *     rollout engine must export its quantization results and the trainer
 *     must consume them.
 *   - aibr.jp/archives/130278, section 3: NVFP4 = blocks of 16 E2M1 values
 *     sharing one E4M3 scale; round-to-nearest forward, stochastic rounding
 *     for backward / weight updates.
 *   - aibr.jp/archives/132665 (TetraJet), section 3: MXFP4 per-group scale.
 *   - "FP4学習の「収縮バイアス」問題を解決するUFP4レシピ" (gotosocial.
 *     chinng-lab-srv.dev), section "UFP4 の設計と実装指針": a uniform 4-bit
 *     grid (E1M2 / INT4) instead of E2M1's.
 *
 * Formats.  E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} indexed by
 * m3 = exponent<<1 | mantissa; a code nibble is sign<<3 | m3.
 *   NVFP4: 16-element blocks along the last dimension; per-segment fp32
 *          tensor scale s_t = amax / (6*448) (below the smallest normal fp32
 *          it is 0 and the segment quantizes to signed zeros); block scale
 *          byte b = E4M3_rne_satfinite( fl32(fl32(bamax/6) / s_t) ); the
 *          block's scale is S = fl32(s_t * E4M3(b)).
 *   MXFP4: 32-element blocks; scale byte = e + 127 with
 *          e = clamp(floor(log2 bamax) - 2, -127, 127) (-127 for an
 *          all-zero block); S = 2^e.  No tensor scale.
 *   UFP4:  the uniform grid {0, 1, ..., 7} (m3 = the magnitude itself) in
 *          NVFP4's container: 16-element blocks, segments, s_t =
 *          amax / (7*448), b = E4M3_rne_satfinite( fl32(fl32(bamax/7) / s_t) ),
 *          S = fl32(s_t * E4M3(b)).  (E1M2's grid is this one / 4; with the
 *          tensor scale taken from the grid maximum both give the same codes
 *          and scale bytes.)  Every rule below reads "the grid maximum" (6 or
 *          7) for 6, and everything the function descriptions say of NVFP4's
 *          s_t, segments and workspace holds for UFP4 too.
 *   Rounding of y = |x| / S (the exact real quotient):
 *     RTN     nearest codeword, ties to even m3, saturating at 6;
 *     SR      between the two neighbours lo < y < hi, round up iff
 *             r < 2^24 (y-lo)/(hi-lo), r = (word 0 of Philox4x32-10 at
 *             counter (i mod 2^32, i >> 32, 0, 0), key (seed mod 2^32,
 *             seed >> 32)) >> 8, i = flat row-major element index within
 *             the call; y >= 6 gives 6, a codeword keeps itself
 *             (Salmon et al., "Parallel random numbers: as easy as 1, 2, 3",
 *             SC'11, defines Philox4x32-10);
 *     guided  of the two neighbours of y, the one whose m3 & 1 equals the
 *             recorded bit; y >= 6 gives 6; a codeword keeps itself;
 *             S == 0 gives signed zero.  The sign is always x's own.
 *
 * Layouts (all contiguous, row-major, flat element index i = r*cols + c):
 *   x         bf16 [rows, cols], cols % 16 == 0 (NVFP4, UFP4) / % 32 (MXFP4)
 *   codes     uint8 [rows*cols/2]; element 2j in the low nibble of byte j
 *   scales    uint8 [rows, cols/block] (linear, not swizzled)
 *   s_t       float [num_segments] (NVFP4 and UFP4 only)
 *   guidance  uint8 [rows*cols/8]; bit (i & 7) of byte (i >> 3) = m3_i & 1
 *
 * Segments.  NVFP4 (and UFP4) may split the rows into num_segments groups (e.g. the
 * per-expert groups of a mixture-of-experts dispatch), each with its own
 * s_t.  seg_row_offsets is a HOST array of num_segments + 1 non-decreasing
 * row offsets, first 0, last rows; empty segments are allowed (their s_t is
 * 0).  NULL means one segment.  MXFP4 requires num_segments == 1.
 *
 * Ownership, streams, errors.  The caller owns every buffer (device memory
 * unless stated) and sizes it as the Layouts above say: the library sees
 * pointers only and cannot check a buffer's extent (the Python binding
 * checks every tensor's size, dtype and device before passing its pointer).
 * The library never allocates, frees or synchronizes,
 * except tf4_read_status, which synchronizes its stream.  Every call is
 * asynchronous on `stream` and launches on the current CUDA device.
 * Argument, shape and alignment problems are returned before anything is
 * launched.  Device pointers must be 16-byte aligned (x, codes, dequant
 * output, unpack output), 4-byte aligned (guidance, s_t, amax, workspace,
 * dev_status); scale arrays have no alignment requirement.
 * Data-dependent problems (a non-finite input) are OR-ed as
 * TF4_DEV_NONFINITE into *dev_status (optional, may be NULL); the outputs
 * of the affected segment (NVFP4 tensor-scale calls) or block are then
 * unspecified.  A failed launch returns TF4_ERR_CUDA.
 *
 * Workspace.  NVFP4 rtn/sr/capture without amax_in, and tf4_segment_amax,
 * need tf4_workspace_bytes(desc) bytes of device workspace that is
 * zero-filled before its first use; each call leaves it zero-filled again
 * when it completes.  Calls that may run concurrently must not share a
 * workspace.
 *
 * Single-launch capture.  An NVFP4 / UFP4 rtn or capture call without
 * amax_in on one segment of at most 2^25 elements (a tensor that fits in
 * half of the L2 cache) runs its amax pass and its quantize pass in one
 * cooperative launch, whose CTAs wait for one another between the two
 * (same results as the two-launch path).  The wait is bounded (100 ms);
 * if it gives up, TF4_DEV_TIMEOUT is OR-ed into *dev_status
 * (tf4_read_status then returns TF4_ERR_TIMEOUT), the call's outputs are
 * unspecified and the workspace is left non-zero: zero-fill it again
 * before reusing it.
 */
#ifndef TRACE_FP4_H
#define TRACE_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* tf4_stream_t;

typedef enum {
  TF4_OK = 0,
  TF4_ERR_INVALID_ARG = 1, /* NULL pointer, bad enum, bad segment offsets */
  TF4_ERR_SHAPE = 2,       /* rows/cols invalid or cols % block != 0       */
  TF4_ERR_ALIGN = 3,       /* pointer misaligned                            */
  TF4_ERR_WORKSPACE = 4,   /* workspace missing or too small                */
  TF4_ERR_NONFINITE = 5,   /* (tf4_read_status) a non-finite input was seen */
  TF4_ERR_TIMEOUT = 6,     /* (tf4_read_status) a bounded device wait gave up */
  TF4_ERR_CUDA = 7         /* a CUDA call failed                            */
} tf4_status;

typedef enum { TF4_NVFP4 = 0, TF4_MXFP4 = 1, TF4_UFP4 = 2 } tf4_format;

#define TF4_MAX_SEGMENTS 1024
#define TF4_MAX_BATCH 64
#define TF4_DEV_NONFINITE 1 /* bit OR-ed into *dev_status */
#define TF4_DEV_TIMEOUT 2   /* bit OR-ed into *dev_status */

typedef struct {
  int32_t fmt;                    /* tf4_format                                */
  int32_t num_segments;           /* >= 1; MXFP4: 1                           */
  int64_t rows;                   /* >= 0                                      */
  int64_t cols;                   /* > 0, multiple of the block size           */
  const int64_t* seg_row_offsets; /* host, num_segments + 1 entries, or NULL  */
} tf4_desc;

/* Sizes in bytes.  record_bytes is the per-call quantization record: codes
 * (with_codes != 0, the full information) or guidance bits (the compact
 * information), plus scale bytes, plus 4 bytes of s_t per segment (NVFP4). */
size_t tf4_workspace_bytes(const tf4_desc* desc);
size_t tf4_codes_bytes(const tf4_desc* desc);
size_t tf4_scales_bytes(const tf4_desc* desc);
size_t tf4_guidance_bytes(const tf4_desc* desc);
size_t tf4_record_bytes(const tf4_desc* desc, int with_codes);

/* NVFP4 segment amax (the grid-wide |x| max pass) on its own: writes
 * amax[num_segments] (device, float).  With several shards of one tensor
 * on several GPUs, an all-reduce MAX of these values followed by
 * quantize calls with amax_in gives every shard the tensor-wide scale.
 * Defined by: the per-tensor fp32 scale of the two-level NVFP4 scaling
 * (aibr.jp/archives/130278, section 3: blocks of 16 share an E4M3 scale;
 * the tensor-level factor amax / (6*448) under it is the format's own). */
tf4_status tf4_segment_amax(const tf4_desc* desc, const void* x, float* amax, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, tf4_stream_t stream);

/* Round-to-nearest quantization.  NVFP4: s_t (device, [num_segments]) is
 * written; amax_in (device, [num_segments], may be NULL) supplies the
 * segment amax and skips the amax pass (no workspace needed).  MXFP4:
 * amax_in, s_t and the workspace are ignored (pass NULL / 0).
 * Defined by: aibr.jp/archives/130278, section 3 (NVFP4 blocks of 16 E2M1
 * values with an E4M3 scale; round-to-nearest in the forward pass);
 * aibr.jp/archives/132665, section 3 (MXFP4's per-group power-of-two
 * scale); the TRACE summary (ai-papers.net), section
 * "学習とロールアウトの不一致": the rollout rounds each value to its nearest
 * codeword. */
tf4_status tf4_quantize_rtn(const tf4_desc* desc, const void* x, const float* amax_in,
                            uint8_t* codes, uint8_t* scales, float* s_t, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, tf4_stream_t stream);

/* Stochastic rounding with the Philox4x32-10 stream keyed by `seed`;
 * otherwise as tf4_quantize_rtn.
 * Defined by: aibr.jp/archives/130278, section 3 (stochastic rounding for
 * the backward pass and weight updates); the random stream is
 * Philox4x32-10 of Salmon et al., "Parallel random numbers: as easy as
 * 1, 2, 3" (SC'11), with the counter and key given under "Rounding" above. */
tf4_status tf4_quantize_sr(const tf4_desc* desc, const void* x, uint64_t seed,
                           const float* amax_in, uint8_t* codes, uint8_t* scales, float* s_t,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status,
                           tf4_stream_t stream);

/* Rollout-side capture: tf4_quantize_rtn plus the compact guidance
 * (m3 & 1 of every element) written to guidance_bits.  Pass
 * guidance_bits = NULL for layers whose guidance is not kept (the caller
 * picks the deepest L of N layers); the codes, scales and s_t are then
 * exactly those of tf4_quantize_rtn.
 * Defined by: the TRACE summary (ai-papers.net), section "TRACEの仕組み"
 * (the rollout records, at every quantization point, the codeword it
 * chose) and section "量子化情報キャッシュ" (only the mantissa bit and the
 * scale are kept, and only for the deeper layers); the Korean explainer
 * (sns.style), section "작동 원리" (the rollout engine exports its
 * quantization results). */
tf4_status tf4_quantize_capture(const tf4_desc* desc, const void* x, const float* amax_in,
                                uint8_t* codes, uint8_t* scales, float* s_t,
                                uint8_t* guidance_bits, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, tf4_stream_t stream);

/* Batched rollout-side capture of num_layers (1..TF4_MAX_BATCH) tensors of
 * the same shape (desc; num_segments must be 1) in two launches instead of
 * two per layer (layers of 2^27 elements or more -- where launch gaps no
 * longer matter -- are run as one launch pair per layer inside the call,
 * with the same results) -- the whole activation stack of a rollout step at once,
 * with the compact records of the deepest `keep` layers written into one
 * contiguous buffer: the quantization-info cache of the TRACE summary's
 * "量子化情報キャッシュ" section, ready to be shipped to the trainer.
 *   x          HOST array [num_layers] of device pointers (16-byte aligned)
 *   codes      device [num_layers][rows*cols/2], contiguous
 *   scales     device [num_layers][rows*cols/block], contiguous
 *   s_t        NVFP4: device [num_layers] (per-layer tensor scale); MXFP4: NULL
 *   keep       0..num_layers: layers [num_layers-keep, num_layers) keep guidance
 *   info_bits  device [keep][rows*cols/8], contiguous (NULL iff keep == 0)
 *   workspace  NVFP4: tf4_workspace_bytes_batched(num_layers) zero-filled bytes
 *              (left zero-filled); MXFP4: unused
 * Per layer the results equal tf4_quantize_capture on that layer alone. */
size_t tf4_workspace_bytes_batched(int32_t num_layers);
tf4_status tf4_quantize_capture_batched(const tf4_desc* desc, int32_t num_layers,
                                        const void* const* x, uint8_t* codes, uint8_t* scales,
                                        float* s_t, int32_t keep, uint8_t* info_bits,
                                        void* workspace, size_t workspace_bytes,
                                        int32_t* dev_status, tf4_stream_t stream);

/* Block scales in the tiled layout block-scaled FP4 GEMMs take for their
 * scale operands (NVIDIA cuBLAS documentation, "1D Block Scaling Factors
 * Layout"; the same bytes a tcgen05 block-scaled MMA's scale tensor holds):
 * the [rows, cols/block] scale matrix, zero-padded to a multiple of 128 rows
 * and 4 columns, as 128 x 4 tiles in row-major tile order, 512 bytes each,
 * entry (r, c) of a tile at byte (r % 32) * 16 + (r / 32) * 4 + c.  NVFP4 /
 * UFP4 scale bytes are the E4M3 block scales (the per-segment s_t stays a
 * separate factor), MXFP4 ones the E8M0 exponents.  The TRACE pages do not
 * define this layout; it lets a captured record feed an FP4 GEMM directly.
 *   scales   device [rows, cols/block] (any alignment)
 *   blocked  device, tf4_blocked_scales_bytes(desc) bytes, 16-byte aligned */
size_t tf4_blocked_scales_bytes(const tf4_desc* desc);
tf4_status tf4_swizzle_scales(const tf4_desc* desc, const uint8_t* scales, uint8_t* blocked,
                              tf4_stream_t stream);

/* Train-side guided quantization of x (the trainer's value) with the
 * rollout's recorded scale bytes, recorded s_t (NVFP4; NULL for MXFP4) and
 * recorded guidance bits.  One pass over x, no workspace.
 * Defined by: the TRACE summary (ai-papers.net), section "TRACEの仕組み":
 * instead of rounding to nearest, the train side takes whichever of the
 * two adjacent codewords matches the rollout's record; section
 * "量子化情報キャッシュ": the mantissa bit and the scale identify it,
 * because mismatches fall between adjacent codewords. */
tf4_status tf4_quantize_guided(const tf4_desc* desc, const void* x, const uint8_t* rec_scales,
                               const float* rec_s_t, const uint8_t* rec_bits, uint8_t* codes,
                               int32_t* dev_status, tf4_stream_t stream);

/* Train-side fake quantization in one pass (the trainer's forward value of
 * the TRACE summary's "mechanism" section: the guided codeword, through
 * which the straight-through gradient flows): tf4_quantize_guided followed
 * by tf4_dequantize, without writing and re-reading the codes.  out
 * receives the dequantized values [rows, cols] as fp32 (out_bf16 = 0) or as
 * bf16, the round-to-nearest-even of that fp32 value (out_bf16 = 1);
 * codes (may be NULL) receives the guided codes.  Alignment: x, out and
 * codes 16 bytes, rec_bits and rec_s_t 4 bytes. */
tf4_status tf4_guided_fake_quant(const tf4_desc* desc, const void* x, const uint8_t* rec_scales,
                                 const float* rec_s_t, const uint8_t* rec_bits, uint8_t* codes,
                                 void* out, int out_bf16, int32_t* dev_status, tf4_stream_t stream);

/* Train/rollout mismatch diagnostics (TRACE summary, section
 * "量子化情報キャッシュ": more than 99% of mismatches fall between adjacent
 * codewords, which is why one mantissa bit suffices, and the corrections
 * toward the smaller codeword concentrate in the deeper layers).  For each
 * element of the train value x, with the rollout's recorded scale bytes /
 * s_t: n_r = nearest rounding of x, n_o = the rollout code (rec_codes), n_g
 * = the guided code (recorded bit = mantissa bit of n_o).  Codes compare by
 * signed grid index (sign ? -m3 : m3; +0 == -0).  ADDS to counts (device,
 * TF4_MISMATCH_COUNTS = 6 x uint64, 8-byte aligned; the caller zeroes it):
 *   counts[0] elements with n_r != n_o, counts[1] with |n_r - n_o| == 1,
 *   counts[2] with |n_r - n_o| >= 2, counts[3] with n_g != n_o,
 *   counts[4] with n_r != n_o and m3(n_o) < m3(n_r) (the rollout's codeword
 *   is the smaller: guidance corrects toward the smaller codeword),
 *   counts[5] with n_r != n_o and m3(n_o) > m3(n_r).
 * (Library version 2; version 1 wrote counts[0..3] only.) */
#define TF4_MISMATCH_COUNTS 6
tf4_status tf4_mismatch_stats(const tf4_desc* desc, const void* x, const uint8_t* rec_scales,
                              const float* rec_s_t, const uint8_t* rec_codes,
                              unsigned long long* counts, int32_t* dev_status, tf4_stream_t stream);

/* out[i] = (-1)^sign * fl32(V[m3] * S) as fp32 [rows, cols].
 * Defined by: the TRACE summary (ai-papers.net), section "TRACEの仕組み":
 * the forward pass carries the chosen quantized value (codeword times its
 * block scale), through which the straight-through gradient flows;
 * aibr.jp/archives/130278, section 3, for the value of an NVFP4 element
 * (E2M1 magnitude times the E4M3 block scale). */
tf4_status tf4_dequantize(const tf4_desc* desc, const uint8_t* codes, const uint8_t* scales,
                          const float* s_t, float* out, tf4_stream_t stream);

/* Guidance extraction from codes produced elsewhere: bits = m3 & 1.
 * Defined by: the TRACE summary (ai-papers.net), section
 * "量子化情報キャッシュ": of the full record only the mantissa bit (with the
 * scale) is sent to the trainer; this packs it from full codes. */
tf4_status tf4_pack_guidance(const tf4_desc* desc, const uint8_t* codes, uint8_t* bits,
                             tf4_stream_t stream);

/* mant[i] = (bits[i >> 3] >> (i & 7)) & 1, one uint8 per element.
 * Defined by: the same section ("量子化情報キャッシュ"): the per-element
 * mantissa bit of the compact record, spread to one byte per element. */
tf4_status tf4_unpack_guidance(const tf4_desc* desc, const uint8_t* bits, uint8_t* mant,
                               tf4_stream_t stream);

/* Allocation-free capture (the paper has no counterpart; this is a library
 * convenience).  Some callers cannot allocate device memory or hand out a
 * workspace: for example a plug-in running inside an engine that owns all
 * device memory, or code on a path where an allocation, which can
 * synchronize the device, is not allowed.  This variant of
 * tf4_quantize_capture takes no workspace: the scratch of its amax pass
 * (num_segments + 1 words) lives in a fixed array of device memory inside
 * the library, which every GPU that loads the library holds until the
 * process exits (1280 bytes per GPU).
 *  - Limit: desc->num_segments <= TF4_NOALLOC_MAX_SEGMENTS, else
 *    TF4_ERR_WORKSPACE is returned and nothing is launched.
 *  - `stream` must belong to the current device (the kernels run there and
 *    use that device's copy of the array); a stream of another device
 *    returns TF4_ERR_INVALID_ARG with nothing launched.
 *  - The first call on a device looks up that device's address of the
 *    array; make that first call before any stream capture.
 *  - Each call clears the scratch it needs (an asynchronous memset on
 *    `stream`) and then behaves exactly like tf4_quantize_capture with
 *    amax_in = NULL.  It calls no cudaMalloc or cudaFree.
 *  - All calls on a device share the one array: calls that may overlap on
 *    the GPU (different streams without ordering) race and must not be
 *    issued; serialize them, or use tf4_quantize_capture with one
 *    workspace per stream. */
#define TF4_NOALLOC_MAX_SEGMENTS 256
tf4_status tf4_quantize_capture_noalloc(const tf4_desc* desc, const void* x, uint8_t* codes,
                                        uint8_t* scales, float* s_t, uint8_t* guidance_bits,
                                        int32_t* dev_status, tf4_stream_t stream);

/* Synchronizes `stream`, reads *dev_status (device), returns TF4_OK,
 * TF4_ERR_NONFINITE, TF4_ERR_TIMEOUT or TF4_ERR_CUDA, and clears it. */
tf4_status tf4_read_status(int32_t* dev_status, tf4_stream_t stream);

const char* tf4_status_string(tf4_status status);
int tf4_version(void);

/* Debug bounds checking (a build option, not part of the method).  A library
 * built with TF4_DEBUG_BOUNDS (python -m fp4_block_scaled_quantizer_b200.build
 * --debug-bounds, which writes libtrace_fp4_debug.so) checks in every kernel
 * that each work unit it reads or writes lies inside the range its CTA owns
 * and inside the buffers' extent; a unit outside is skipped and counted in a
 * library-wide device counter instead of being accessed (no trap).
 *   tf4_debug_bounds_enabled: 1 for such a build, 0 otherwise.
 *   tf4_debug_bounds_violations: synchronizes `stream`, writes the number of
 *     skipped units counted since the last call (on the current device) to
 *     *count (host pointer) and resets the counter; always 0 in a build
 *     without the checks.  Returns TF4_OK, TF4_ERR_INVALID_ARG (count NULL)
 *     or TF4_ERR_CUDA. */
int tf4_debug_bounds_enabled(void);
tf4_status tf4_debug_bounds_violations(uint64_t* count, tf4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRACE_FP4_H */
