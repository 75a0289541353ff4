/*
 * tf4_oracle.h -- plain CPU oracle for block-scaled FP4 quantization.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline / reference leg of bench.py may
 * load this library.  It shares no code, header, table or helper with the
 * CUDA library under fp4_block_scaled_quantizer_b200/csrc.
 *
 * Sources followed (web pages, cited by title and section):
 *   [TRACE-JA]  "TRACE: Rollout-Guided Quantization-Aware Training for FP4
 *               Reinforcement Learning of MoE Language Models", summary at
 *               ai-papers.net; sections "学習とロールアウトの不一致" (train /
 *               rollout mismatch), "TRACEの仕組み" (mechanism),
 *               "量子化情報キャッシュ" (quantization-info cache).
 *   [TRACE-KO]  Korean explainer of the same paper (sns.style), sections
 *               "핵심 아이디어" and "작동 원리".
 *   [FQT]       aibr.jp/archives/130278, section 3 (core techniques):
 *               NVFP4 = 16-value blocks of E2M1 sharing one E4M3 scale;
 *               round-to-nearest forward, stochastic rounding backward.
 *   [TETRAJET]  aibr.jp/archives/132665, section 3: MXFP4 per-group scale.
 *   [UFP4]      "FP4学習の「収縮バイアス」問題を解決するUFP4レシピ" (gotosocial.
 *               chinng-lab-srv.dev), section "UFP4 の設計と実装指針": a
 *               uniform 4-bit grid (E1M2 / INT4) in place of E2M1.
 *   [PHILOX]    Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *               easy as 1, 2, 3", SC'11 -- the Philox4x32-10 generator.
 *   [CUBLAS]    NVIDIA cuBLAS documentation, "1D Block Scaling Factors
 *               Layout" -- the tiled scale layout of block-scaled GEMMs
 *               (not on the TRACE pages; used by orc_swizzle_scales).
 *
 * Layouts (identical to the library's public layouts, restated here):
 *   x        bf16 bit patterns, row-major [rows, cols], cols % block == 0
 *   codes    packed E2M1 nibbles, 2 per byte, element 2j in the low nibble;
 *            nibble = sign<<3 | m3, m3 indexes {0,.5,1,1.5,2,3,4,6}
 *   scales   one byte per block, row-major [rows, cols/block]
 *            NVFP4 / UFP4: E4M3 (fn) code; MXFP4: E8M0 byte = exponent + 127
 *   s_t      NVFP4 / UFP4 only: one fp32 per segment (per-tensor scale)
 *
 * Formats: NVFP4 = E2M1 grid, 16-element blocks, E4M3 scale, fp32 s_t;
 * MXFP4 = E2M1 grid, 32-element blocks, E8M0 scale; UFP4 = the uniform grid
 * {0,1,...,7} in NVFP4's container (16-element blocks, E4M3 scale, fp32
 * s_t = amax / (7 * 448)).
 *   bits     guidance: bit (i&7) of byte (i>>3) = m3_i & 1, i = flat index
 *
 * Return values: 0 = ok, otherwise a bitmask; bit 0 (ORC_NONFINITE) means a
 * non-finite input was seen (outputs of the affected segment (NVFP4) or
 * block (MXFP4) are then unspecified).
 */
#ifndef TF4_ORACLE_H
#define TF4_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_NVFP4 0
#define ORC_MXFP4 1
#define ORC_UFP4 2
#define ORC_RTN 0
#define ORC_SR 1
#define ORC_NONFINITE 1

/* element-level definitions (exported so that tests can pin them) */
float orc_bf16_to_float(uint16_t h);
double orc_e2m1_value(int m3);
double orc_grid_value(int fmt, int m3);
double orc_e4m3_value(uint8_t code);
uint8_t orc_e4m3_encode(float r);
int orc_e8m0_exponent(float bamax);
float orc_tensor_scale(int fmt, float amax);
float orc_nvfp4_tensor_scale(float amax);
uint8_t orc_block_scale_code(int fmt, float bamax, float s_t);
uint8_t orc_nvfp4_block_scale_code(float bamax, float s_t);
float orc_nvfp4_block_scale(uint8_t code, float s_t);
float orc_mxfp4_block_scale(uint8_t code);
int orc_rtn_m3(double ax, double S);
int orc_sr_m3(double ax, double S, uint32_t r24);
int orc_guided_m3(double ax, double S, int g);
int orc_rtn_code(int fmt, double ax, double S);
int orc_sr_code(int fmt, double ax, double S, uint32_t r24);
int orc_guided_code(int fmt, double ax, double S, int g);
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
uint32_t orc_sr_uniform24(uint64_t idx, uint64_t seed);

/* tensor-level definitions */
int orc_segment_amax(const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                     const int64_t* seg_off, float* amax_out);
int orc_segment_scales(int fmt, const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                       const int64_t* seg_off, float* s_t_out);
int orc_quantize_rows(int fmt, int mode, const uint16_t* x, int64_t rows, int64_t cols,
                      int32_t nseg, const int64_t* seg_off, const float* s_t, uint64_t seed,
                      int64_t row_begin, int64_t row_end, uint8_t* codes, uint8_t* scales,
                      uint8_t* bits);
int orc_quantize_guided_rows(int fmt, const uint16_t* x, int64_t rows, int64_t cols,
                             int32_t nseg, const int64_t* seg_off, const uint8_t* rec_scales,
                             const float* rec_s_t, const uint8_t* rec_bits, int64_t row_begin,
                             int64_t row_end, uint8_t* codes);
void orc_dequantize_rows(int fmt, const uint8_t* codes, const uint8_t* scales, const float* s_t,
                         int64_t rows, int64_t cols, int32_t nseg, const int64_t* seg_off,
                         int64_t row_begin, int64_t row_end, float* out);
void orc_pack_guidance(const uint8_t* codes, int64_t n, uint8_t* bits);
void orc_unpack_guidance(const uint8_t* bits, int64_t n, uint8_t* mant);
void orc_rtn_with_scales_rows(int fmt, const uint16_t* x, int64_t rows, int64_t cols, int32_t nseg,
                              const int64_t* seg_off, const uint8_t* scales, const float* s_t,
                              int64_t row_begin, int64_t row_end, uint8_t* codes);
void orc_swizzle_scales(const uint8_t* scales, int64_t rows, int64_t nb, uint8_t* out);
uint16_t orc_f32_to_bf16(float v);
void orc_f32_to_bf16_array(const float* v, int64_t n, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
