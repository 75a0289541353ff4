// tf4_kernels.cuh -- sm_100a kernels of the trace_fp4 library.
//
// Streaming, elementwise + reduction work: no tensor cores.  Every kernel
// splits its flat array of quantization blocks into one contiguous range
// per CTA (grid = 1 to 4 waves of SMs x resident CTAs, chosen on the host),
// and lanes of a warp take consecutive work units so that each warp
// instruction moves a contiguous span.  Quantize / guided passes: one lane
// owns one block per unit (NVFP4 / UFP4: 16 elements, 32 B of bf16, two
// 16-B loads; MXFP4: 32 elements, four loads); the fused fake-quant and the
// wide-store dequantize take 8 elements per lane, the narrow-store
// dequantize 4.
//
// Definitions followed are stated in include/trace_fp4.h (and the pages
// cited there); the notes below only explain how each kernel reaches the
// exact definition.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "../../include/trace_fp4.h"

namespace tf4 {

constexpr int kThreads = 256;

// Formats with an E4M3 block scale and an fp32 tensor scale (16-element
// blocks, segments): NVFP4 (E2M1 grid) and UFP4 (uniform grid 0..7).
template <int FMT>
constexpr bool kE4M3 = FMT != TF4_MXFP4;
template <int FMT>
constexpr bool kUni = FMT == TF4_UFP4;
// Largest grid value (6 on E2M1, 7 on the uniform grid): the block-scale
// divisor, and 448 times it is the tensor-scale divisor.
template <bool U>
constexpr float kGridMax = U ? 7.0f : 6.0f;

// Programmatic dependent launch.  The library launches its kernels with
// programmatic stream serialization, so a kernel may be scheduled while the
// grid before it in the stream is still finishing.  Every kernel therefore
// first waits for that grid to complete and its memory to be visible
// (before reading or writing anything), then lets the next grid begin
// launching.  Without the launch attribute both instructions are no-ops.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// First unit of part i when n units are split into `grid` parts whose
// sizes differ by at most one (part i is [cta_begin(i), cta_begin(i + 1))).
__device__ __forceinline__ int64_t cta_begin(int64_t i, int64_t grid, int64_t n) {
  const int64_t q = n / grid, r = n % grid;
  return i * q + (i < r ? i : r);
}

// ------------------------------------------------------------- segments
// One per-tensor-scale segment covering everything (the common case).
struct Seg1 {
  __device__ __forceinline__ int find(int64_t /*block*/) const { return 0; }
  __device__ __forceinline__ int64_t start(int /*s*/) const { return 0; }
  __device__ __forceinline__ int count() const { return 1; }
  // input / guidance base pointers of segment s, addressed by the global
  // block index (one tensor: the call's own pointers)
  __device__ __forceinline__ const uint4* xptr(int /*s*/, const uint4* x) const { return x; }
  __device__ __forceinline__ uint8_t* bitsptr(int /*s*/, uint8_t* b) const { return b; }
};

// Ragged segments (row offsets, passed by value in the kernel parameters).
struct SegN {
  int32_t nseg;
  int64_t bpr;  // quantization blocks per row
  int32_t off[TF4_MAX_SEGMENTS + 1];
  // The segment holding `block`: the largest s with off[s] <= row (it is
  // then non-empty).
  __device__ __forceinline__ int find(int64_t block) const {
    const int64_t row = block / bpr;
    int lo = 0, hi = nseg;  // answer in [lo, hi)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= row) lo = mid; else hi = mid;
    }
    return lo;
  }
  __device__ __forceinline__ int64_t start(int s) const { return (int64_t)off[s] * bpr; }
  __device__ __forceinline__ int count() const { return nseg; }
  __device__ __forceinline__ const uint4* xptr(int /*s*/, const uint4* x) const { return x; }
  __device__ __forceinline__ uint8_t* bitsptr(int /*s*/, uint8_t* b) const { return b; }
};

// Ragged segments with one piece per CTA (the guided kernels): the host
// gives each non-empty segment its own CTAs (cta[s] .. cta[s+1] - 1, about
// in proportion to its blocks), so no CTA walks from one segment into the
// next; that walk, carried in registers around two instantiations of the
// block loop, made the loop spill.
struct SegPieces {
  int32_t nseg;
  int64_t bpr;                         // quantization blocks per row
  int32_t off[TF4_MAX_SEGMENTS + 1];   // row offsets of the segments
  int32_t cta[TF4_MAX_SEGMENTS + 1];   // first CTA of each segment (non-decreasing; cta[nseg] = grid)
  // CTA i's segment s (the largest s with cta[s] <= i: non-empty) and its
  // part [lo, hi), part i - cta[s] of cta[s+1] - cta[s] near-equal parts.
  __device__ __forceinline__ void piece(int i, int& s, int64_t& lo, int64_t& hi) const {
    int l = 0, h = nseg;  // answer in [l, h)
    while (h - l > 1) {
      const int mid = (l + h) >> 1;
      if (cta[mid] <= i) l = mid; else h = mid;
    }
    s = l;
    const int64_t b = (int64_t)off[l] * bpr, e = (int64_t)off[l + 1] * bpr;
    const int k = i - cta[l], cnt = cta[l + 1] - cta[l];
    lo = b + cta_begin(k, cnt, e - b);
    hi = b + cta_begin(k + 1, cnt, e - b);
  }
};

// A batch of same-shaped tensors (layers) quantized by one launch: segment s
// is layer s with its own input pointer and its own tensor scale; codes and
// scales are contiguous across layers (global block index), guidance bits
// are kept only for layers s >= first_kept and stored contiguously from
// there (the info cache).  The returned bases are offset so that
// base + (units per block) * global_block addresses the layer's data.
struct SegBatch {
  int32_t nlayers;
  int32_t first_kept;       // layers >= first_kept write guidance
  int64_t bpl;              // blocks per layer
  int32_t units_per_block;  // 16-byte input units per block (2 NVFP4, 4 MXFP4)
  int32_t bits_per_block;   // guidance bytes per block (2 NVFP4, 4 MXFP4)
  const uint4* x[TF4_MAX_BATCH];
  __device__ __forceinline__ int find(int64_t block) const { return (int)(block / bpl); }
  __device__ __forceinline__ int64_t start(int s) const { return (int64_t)s * bpl; }
  __device__ __forceinline__ int count() const { return nlayers; }
  __device__ __forceinline__ const uint4* xptr(int s, const uint4*) const {
    return reinterpret_cast<const uint4*>(reinterpret_cast<uintptr_t>(x[s]) -
                                          (uintptr_t)(start(s) * units_per_block * 16));
  }
  __device__ __forceinline__ uint8_t* bitsptr(int s, uint8_t* b) const {
    if (!b || s < first_kept) return nullptr;
    return reinterpret_cast<uint8_t*>(reinterpret_cast<uintptr_t>(b) -
                                      (uintptr_t)(start(first_kept) * bits_per_block));
  }
};

// ------------------------------------------------------- debug bounds
// Builds with TF4_DEBUG_BOUNDS check every work unit a kernel is about to
// read or write: its index must lie in the range [lo, hi) the CTA is
// working on and in [0, n), the extent of the buffers in those units.  A
// unit outside is skipped (not read, not written) and counted in
// g_tf4_bounds, which tf4_debug_bounds_violations reads and clears.  In
// other builds the check is the constant true and compiles away.
__device__ unsigned long long g_tf4_bounds;

__device__ __forceinline__ bool unit_ok(int64_t i, int64_t lo, int64_t hi, int64_t n) {
#ifdef TF4_DEBUG_BOUNDS
  if (i >= lo && i < hi && i >= 0 && i < n) return true;
  atomicAdd(&g_tf4_bounds, 1ull);
  return false;
#else
  (void)i; (void)lo; (void)hi; (void)n;
  return true;
#endif
}

// ---------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// bf16 pair -> two fp32 (exact widening)
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per half of two bf16 pairs: the larger magnitude (the sign bits are the
// XOR of the inputs' and get masked off by the caller), NaN if either is
// NaN.  Comparing bf16 values is exact.
__device__ __forceinline__ uint32_t hmax_abs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Max |x| over words of bf16 pairs, as a bf16 bit pattern (0x7F80 or more
// means a non-finite input: the magnitude bit order is the value order).
template <int N>
__device__ __forceinline__ uint32_t block_absmax_bits(const uint32_t (&w)[N]) {
  uint32_t m = w[0];
#pragma unroll
  for (int i = 1; i < N; ++i) m = hmax_abs(m, w[i]);
  m &= 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

// Eight fp32 values -> eight E2M1 nibbles (hardware RNE, satfinite),
// element k in bits [4k, 4k+4).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                               float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// Eight fp32 values -> eight E2M3 codes (hardware RNE, satfinite): element
// k in byte k & 3 of b[k >> 2], each byte s << 5 | e << 3 | m.
__device__ __forceinline__ void cvt_e2m3x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7, uint32_t& b0, uint32_t& b1) {
  asm("{\n\t.reg .b16 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 q0, %3, %2;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 q1, %5, %4;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 q2, %7, %6;\n\t"
      "cvt.rn.satfinite.e2m3x2.f32 q3, %9, %8;\n\t"
      "mov.b32 %0, {q0, q1};\n\t"
      "mov.b32 %1, {q2, q3};\n\t}"
      : "=r"(b0), "=r"(b1)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
}


// Eight fp32 values -> eight uniform-grid nibbles: round |v| to the nearest
// integer, ties to even (adding 2^23 does exactly that: the sum is rounded
// once, to a neighbouring integer), saturating at 7; sign bit kept.  Element
// k in bits [4k, 4k+4).
__device__ __forceinline__ uint32_t cvt_uni_x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                               float v6, float v7) {
  const float v[8] = {v0, v1, v2, v3, v4, v5, v6, v7};
  uint32_t r = 0u;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t t = __float_as_uint(__fadd_rn(fminf(fabsf(v[k]), 7.0f), 0x1p23f));
    r |= ((t & 7u) | ((__float_as_uint(v[k]) >> 28) & 8u)) << (4 * k);
  }
  return r;
}

// Eight fp32 values -> eight nibbles of the format's grid.
template <bool U>
__device__ __forceinline__ uint32_t cvt_grid_x8(float v0, float v1, float v2, float v3, float v4, float v5,
                                                float v6, float v7) {
  if constexpr (U) return cvt_uni_x8(v0, v1, v2, v3, v4, v5, v6, v7);
  else return cvt_e2m1x8(v0, v1, v2, v3, v4, v5, v6, v7);
}

// Four E2M1 nibbles (16 bits, element k in bits [4k, 4k+4)) -> their values
// times S, using CUDA's fp4x2 -> half2 conversion (exact: every E2M1 value
// is an f16 value) and one fp32 multiply each.
__device__ __forceinline__ float4 decode4(uint32_t c, float S) {
  const __half2_raw h0 = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(c & 0xFFu), __NV_E2M1);
  const __half2_raw h1 = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)((c >> 8) & 0xFFu), __NV_E2M1);
  const float2 f0 = __half22float2(__half2(h0));
  const float2 f1 = __half22float2(__half2(h1));
  return make_float4(__fmul_rn(f0.x, S), __fmul_rn(f0.y, S), __fmul_rn(f1.x, S), __fmul_rn(f1.y, S));
}

// Four uniform-grid nibbles -> +-RN(k * S); k as fp32 via 2^23 + k - 2^23.
__device__ __forceinline__ float4 decode4_uni(uint32_t c, float S) {
  float v[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t n = (c >> (4 * e)) & 0xFu;
    const float k = __fsub_rn(__uint_as_float(0x4B000000u | (n & 7u)), 0x1p23f);
    v[e] = __uint_as_float(__float_as_uint(__fmul_rn(k, S)) | ((n & 8u) << 28));
  }
  return make_float4(v[0], v[1], v[2], v[3]);
}

// The same through CUDA's E4M3 -> half conversion: magnitude k (0..7) as an
// E4M3 byte is the subnormal k * 2^-9 (exact in f16), the nibble's sign
// goes to the byte's sign bit, and (k 2^-9) (S 2^9) = k S is rounded once.
// Needs S 2^9 finite: the caller checks S <= 2^100.
__device__ __forceinline__ float4 decode4_uni_e4m3(uint32_t c, float S) {
  uint32_t t = c & 0xFFFFu;
  t = (t | (t << 8)) & 0x00FF00FFu;   // n0|n1<<4 in byte 0, n2|n3<<4 in byte 2
  t = (t | (t << 4)) & 0x0F0F0F0Fu;   // n0..n3 in bytes 0..3
  t = (t & 0x07070707u) | ((t & 0x08080808u) << 4);
  const float S9 = S * 512.0f;        // exact
  const __half2_raw h0 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(t & 0xFFFFu), __NV_E4M3);
  const __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(t >> 16), __NV_E4M3);
  const float2 f0 = __half22float2(__half2(h0));
  const float2 f1 = __half22float2(__half2(h1));
  return make_float4(__fmul_rn(f0.x, S9), __fmul_rn(f0.y, S9), __fmul_rn(f1.x, S9), __fmul_rn(f1.y, S9));
}

template <bool U>
__device__ __forceinline__ float4 decode4_grid(uint32_t c, float S) {
  if constexpr (U) return S <= 0x1p100f ? decode4_uni_e4m3(c, S) : decode4_uni(c, S);
  else return decode4(c, S);
}

// Eight nibbles (a code word) -> v0 (elements 0..3), v1 (4..7), as
// decode4_grid twice; on the uniform grid the nibbles are spread to bytes
// for all eight at once (byte_perm of the even and odd nibbles).
template <bool U>
__device__ __forceinline__ void decode8_grid(uint32_t c, float S, float4& v0, float4& v1) {
  if constexpr (U) {
    if (S <= 0x1p100f) {
      const uint32_t lo = c & 0x0F0F0F0Fu, hi = (c >> 4) & 0x0F0F0F0Fu;  // nibbles 0,2,4,6 / 1,3,5,7
      uint32_t p[2] = {__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362)};
      const float S9 = S * 512.0f;  // exact
      float4 v[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        p[h] = (p[h] & 0x07070707u) | ((p[h] & 0x08080808u) << 4);
        const __half2_raw h0 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(p[h] & 0xFFFFu), __NV_E4M3);
        const __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(p[h] >> 16), __NV_E4M3);
        const float2 f0 = __half22float2(__half2(h0));
        const float2 f1 = __half22float2(__half2(h1));
        v[h] = make_float4(__fmul_rn(f0.x, S9), __fmul_rn(f0.y, S9), __fmul_rn(f1.x, S9), __fmul_rn(f1.y, S9));
      }
      v0 = v[0];
      v1 = v[1];
      return;
    }
  }
  v0 = decode4_grid<U>(c & 0xFFFFu, S);
  v1 = decode4_grid<U>(c >> 16, S);
}

// One 32-byte store (sm_100 256-bit vector store); p must be 32-B aligned.
__device__ __forceinline__ void st_v8(float* p, const float4& a, const float4& b) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(a.x), "f"(a.y), "f"(a.z),
               "f"(a.w), "f"(b.x), "f"(b.y), "f"(b.z), "f"(b.w)
               : "memory");
}

// m3 & 1 of eight nibbles -> eight bits (nibble k -> bit k).  The masked
// bits sit at 4k; multiplying by 0x1248 (= 2^3 + 2^6 + 2^9 + 2^12) sends bit
// 4k to 12 + k for k < 4 and to 24 + k for k >= 4, and every other partial
// product lands on a distinct position outside those bits (no carries).
__device__ __forceinline__ uint32_t nibble_lsbs(uint32_t c) {
  const uint32_t p = (c & 0x11111111u) * 0x1248u;
  return ((p >> 12) & 0xFu) | ((p >> 24) & 0xF0u);
}

// E4M3 (fn) scale byte of a non-negative fp32 (hardware RNE, satfinite).
__device__ __forceinline__ uint32_t e4m3_encode(float r) {
  return (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
}

// Value of an E4M3 byte in [0, 0x7E].
__device__ __forceinline__ float e4m3_decode(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  if (e == 0) return (float)m * 0x1p-9f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Per-tensor scale from the segment amax, amax / (448 * grid max)
// (2688 for E2M1, 3136 for the uniform grid); non-finite amax -> NaN.
template <bool U = false>
__device__ __forceinline__ float tensor_scale(float amax, int32_t* status) {
  if (!(amax <= 3.4028234663852886e38f)) {  // Inf or NaN
    if (status) atomicOr(status, TF4_DEV_NONFINITE);
    return __int_as_float(0x7FC00000);
  }
  const float s = __fdiv_rn(amax, 448.0f * kGridMax<U>);
  return s >= 0x1p-126f ? s : 0.0f;
}

// A value within 8 fp32 ulps of a bf16 number (low 16 bits near 0 or 2^16).
__device__ __forceinline__ bool near_bf16(float v) {
  return ((__float_as_uint(v) + 8u) & 0xFFFFu) < 16u;
}

// ------------------------------------------------------------ grid values
// Magnitude of E2M1 code m3 (0..7) as fp32.
__device__ __forceinline__ float e2m1_value(uint32_t m3) {
  const uint32_t e = m3 >> 1, m = m3 & 1u;
  return e ? __uint_as_float(((e + 126u) << 23) | (m << 22)) : (m ? 0.5f : 0.0f);
}

// Magnitude of code m3 on the format's grid (uniform: m3 itself).
template <bool U>
__device__ __forceinline__ float grid_value(uint32_t m3) {
  if constexpr (U) return (float)m3;
  else return e2m1_value(m3);
}

// Midpoint between codes i and i + 1.
template <bool U>
__device__ __forceinline__ float grid_mid(int i) {
  return 0.5f * (grid_value<U>((uint32_t)i) + grid_value<U>((uint32_t)i + 1u));
}

// ------------------------------------------------- exact per-element paths
// RTN m3 of |x| on scale S > 0 by exact comparisons.  fmaf(-mu, S, ax) is
// rounded once, so its sign is the sign of ax - mu*S exactly as long as the
// difference cannot underflow, which holds for S >= 2^-124; smaller S is
// rescaled by 2^64 first (exact).  Three-level search over the 7 midpoints
// (E2M1: .25,.75,1.25,1.75,2.5,3.5,5; uniform: .5, 1.5, ..., 6.5); ">=" at
// odd-index midpoints and ">" at even-index ones give ties to the even m3.
template <bool U = false>
__device__ __forceinline__ uint32_t rtn_m3_exact(float ax, float S) {
  if (S < 0x1p-100f) {
    ax *= 0x1p64f;
    S *= 0x1p64f;
  }
  const bool b2 = fmaf(-grid_mid<U>(3), S, ax) >= 0.0f;
  const float mu = b2 ? grid_mid<U>(5) : grid_mid<U>(1);
  const bool b1 = fmaf(-mu, S, ax) >= 0.0f;
  const float mu3 = b2 ? (b1 ? grid_mid<U>(6) : grid_mid<U>(4)) : (b1 ? grid_mid<U>(2) : grid_mid<U>(0));
  const bool b0 = fmaf(-mu3, S, ax) > 0.0f;
  return (b2 ? 4u : 0u) | (b1 ? 2u : 0u) | (b0 ? 1u : 0u);
}

// Guided m3 of |x| on scale S > 0 with recorded bit g (exact comparisons as
// above): f = number of nonzero codewords <= y; y >= grid max -> 7; y a
// codeword -> f; otherwise the neighbour (f or f+1) whose m3 & 1 == g.
template <bool U = false>
__device__ __forceinline__ uint32_t guided_m3_exact(float ax, float S, uint32_t g) {
  if (S < 0x1p-100f) {
    ax *= 0x1p64f;
    S *= 0x1p64f;
  }
  const float d2 = fmaf(-grid_value<U>(4), S, ax);
  const bool p2 = d2 >= 0.0f;
  const float v1 = p2 ? grid_value<U>(6) : grid_value<U>(2);
  const float d1 = fmaf(-v1, S, ax);
  const bool p1 = d1 >= 0.0f;
  const float v0 = p2 ? (p1 ? grid_value<U>(7) : grid_value<U>(5)) : (p1 ? grid_value<U>(3) : grid_value<U>(1));
  const float d0 = fmaf(-v0, S, ax);
  const bool p0 = d0 >= 0.0f;
  const uint32_t f = (p2 ? 4u : 0u) | (p1 ? 2u : 0u) | (p0 ? 1u : 0u);
  const bool exact = p0 ? (d0 == 0.0f) : p1 ? (d1 == 0.0f) : p2 ? (d2 == 0.0f) : (ax == 0.0f);
  if (f == 7u || exact) return f;
  return f + ((f ^ g) & 1u);
}

// Philox4x32-10 (Salmon et al., SC'11), word 0 only, counter
// (idx mod 2^32, idx >> 32, 0, 0), key = seed.  One round maps
// (c0, c1, c2, c3) to (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1,
// lo(M0 c0)); round j (0..9) uses the key (k0 + j W0, k1 + j W1).  The
// quantize kernels take that schedule as kernel parameters (ks[2j],
// ks[2j+1]) so the round keys are constant-bank operands.  Elements of one
// quantization block share idx >> 32 (blocks of 16 or 32 never straddle a
// multiple of 2^32), which makes round 2's M0 product the same for the
// whole block (PhiloxBlk).  With the zero words of the counter, round 1 has
// one product, and round 10 needs only hi(M1 c2) for word 0.
constexpr uint32_t kPhiloxM0 = 0xD2511F53u, kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u, kPhiloxW1 = 0xBB67AE85u;
constexpr int kPhiloxKeys = 20;

__device__ __forceinline__ void mulhilo(uint32_t m, uint32_t c, uint32_t& hi, uint32_t& lo) {
  const uint64_t p = (uint64_t)m * c;
  hi = (uint32_t)(p >> 32);
  lo = (uint32_t)p;
}

struct PhiloxBlk {
  uint32_t c1;        // idx >> 32 of the block
  uint32_t hi2, lo2;  // round 2: M0 * (c1 ^ k0)
};

__device__ __forceinline__ PhiloxBlk philox_block(uint64_t first_idx, const uint32_t* ks) {
  PhiloxBlk b;
  b.c1 = (uint32_t)(first_idx >> 32);
  mulhilo(kPhiloxM0, b.c1 ^ ks[0], b.hi2, b.lo2);
  return b;
}

// Word 0 for counter (lo32, b.c1, 0, 0) under key schedule ks.
__device__ __forceinline__ uint32_t philox_w0_blk(uint32_t lo32, const PhiloxBlk& b, const uint32_t* ks) {
  uint32_t hi0, lo0, hi1, lo1;
  // round 1 (c2 = c3 = 0, so M1 c2 = 0): c0 <- c1_in ^ k0, whose M0 product
  // is the block's (b.hi2, b.lo2); c1 <- 0; c2, c3 from M0 lo32
  mulhilo(kPhiloxM0, lo32, hi0, lo0);
  uint32_t c2 = hi0 ^ ks[1], c3 = lo0;
  // round 2
  mulhilo(kPhiloxM1, c2, hi1, lo1);
  uint32_t c0 = hi1 ^ ks[2];  // ^ c1, which is 0
  uint32_t c1 = lo1;
  c2 = b.hi2 ^ c3 ^ ks[3];
  c3 = b.lo2;
#pragma unroll
  for (int j = 2; j < 9; ++j) {
    mulhilo(kPhiloxM0, c0, hi0, lo0);
    mulhilo(kPhiloxM1, c2, hi1, lo1);
    c0 = hi1 ^ c1 ^ ks[2 * j];
    c1 = lo1;
    c2 = hi0 ^ c3 ^ ks[2 * j + 1];
    c3 = lo0;
  }
  // round 10: word 0 only
  return __umulhi(kPhiloxM1, c2) ^ c1 ^ ks[18];
}

// The key schedule of a seed (host and device).
__host__ __device__ inline void philox_schedule(uint64_t seed, uint32_t (&ks)[kPhiloxKeys]) {
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int j = 0; j < 10; ++j) {
    ks[2 * j] = k0;
    ks[2 * j + 1] = k1;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
}

// Word 0 for counter (idx mod 2^32, idx >> 32, 0, 0), key = seed.
__device__ __forceinline__ uint32_t philox_w0(uint64_t idx, uint64_t seed) {
  uint32_t ks[kPhiloxKeys];
  philox_schedule(seed, ks);
  return philox_w0_blk((uint32_t)idx, philox_block(idx, ks), ks);
}

// SR m3 of |x| on scale S > 0 with a 24-bit uniform r.  Every product of a
// codeword (<= 4 significant bits) and S (24 bits) is exact in double, and
// so are r * gap * S (<= 48 bits) and ax - V_lo * S (V_lo = 0, or
// ax >= S/2 ends at or above bit 2^-8 S while V_lo * S ends at or above
// 2^-25 S and both are below 2^4 S), so all comparisons are exact.
template <bool U = false>
__device__ __forceinline__ uint32_t sr_m3_exact(float axf, float Sf, uint32_t r24) {
  const double ax = axf, S = Sf;
  if (ax >= (double)kGridMax<U> * S) return 7u;
  // f = number of nonzero codewords <= y
  uint32_t f = 0u;
#pragma unroll
  for (uint32_t j = 1; j < 8; ++j) f += (double)grid_value<U>(j) * S <= ax;
  const double vlo = (double)grid_value<U>(f), vhi = (double)grid_value<U>(f + 1u);
  if (vlo * S == ax) return f;
  const double lhs = (double)r24 * (vhi - vlo) * S;
  const double rhs = 16777216.0 * (ax - vlo * S);
  return lhs < rhs ? f + 1u : f;
}

// Stochastic rounding on the E2M1 grid from the exact quotient y = |x| / S
// (MXFP4: a power-of-two scale): lo and gap come from the fp32 bits of y
// (for y >= 1 the grid is the 1-mantissa-bit truncation, gap 2^(E-1); below
// 1 it is {0, 0.5} with gap 0.5), and t = 2^24 (y - lo) / gap is exact
// arithmetic on y (Sterbenz subtraction, power-of-two scaling), so r24 < t
// decides exactly.  Returns the chosen codeword value.
__device__ __forceinline__ float sr_pick_e2m1_exact(float y, uint32_t r24) {
  const uint32_t yb = __float_as_uint(y);
  const bool ge1 = y >= 1.0f;
  const float vlo = ge1 ? __uint_as_float(yb & 0xFFC00000u) : (y >= 0.5f ? 0.5f : 0.0f);
  const float gap = ge1 ? __uint_as_float((yb & 0x7F800000u) - 0x00800000u) : 0.5f;
  const float inv = ge1 ? __uint_as_float((279u - (yb >> 23)) << 23) : 0x1p25f;  // 2^24 / gap
  const float t = __fmul_rn(__fsub_rn(y, vlo), inv);
  const float v = __uint2float_rn(r24) < t ? __fadd_rn(vlo, gap) : vlo;  // r24 < 2^24: exact
  return fminf(v, 6.0f);
}

// Stochastic rounding on the uniform grid from y = |x| / S given as a
// product that is on the correct side of every codeword and equals one iff
// y does: lo = floor(y), gap 1, and t = 2^24 (y - lo) is exact arithmetic on
// y (Sterbenz subtraction).  |y - y_exact| < 2^-17.5 for y < 7.5, so
// |t - T_exact| < 96 and a uniform within 128 of t is flagged `amb` for the
// exact test.  Returns the chosen codeword value (saturated at 7).
__device__ __forceinline__ float sr_pick_uni(float y, uint32_t r24, bool& amb) {
  const float vlo = floorf(y);
  const float t = __fmul_rn(__fsub_rn(y, vlo), 0x1p24f);
  const float rf = __uint2float_rn(r24);  // exact: r24 < 2^24
  amb = fabsf(rf - t) <= 128.0f;
  const float v = rf < t ? __fadd_rn(vlo, 1.0f) : vlo;
  return fminf(v, 7.0f);
}

// Stochastic rounding on the E2M1 grid from y2 = 2y (y = |x| / S given
// exactly, or as a product on the correct side of every codeword) and the
// Philox word pw.  W = max(2y, RZ(y + 1)) maps the grid {0, .5, 1, 1.5, 2,
// 3, 4, 6} onto the numbers with one mantissa bit {1, 1.5, 2, 3, 4, 6, 8,
// 12} (W = 2y for y >= 1, y + 1 below), so the code of lo is
// (bits(W) >> 22) - 254 and the threshold 2^24 (y - lo) / (hi - lo) is
// 4 (bits(W) & 0x3FFFFF), four times the mantissa bits below the top one:
// round up iff r24 = pw >> 8 is below it, i.e. iff pw >> 10 is below
// bits(W) & 0x3FFFFF.  RZ(y + 1) (error < 2^-23) and an approximate y move
// the threshold by less than 64, so a uniform within 128 of it is flagged
// `amb` for the exact test.  Returns m3, saturated at 7 (y >= 6, and any
// huge y, map to code 7 or above before the cap).
__device__ __forceinline__ uint32_t sr_e2m1(float y2, uint32_t pw, bool& amb) {
  const uint32_t wb = __float_as_uint(fmaxf(y2, __fmaf_rz(y2, 0.5f, 1.0f)));
  const uint32_t m = wb & 0x3FFFFFu;
  amb = (pw >> 8) - (m << 2) + 128u <= 256u;
  return min((wb >> 22) - 254u + ((pw >> 10) < m ? 1u : 0u), 7u);
}

// -------------------------------------------------------------- amax pass
// Grid-wide max |x| per segment.  Each CTA reduces its range piece by
// piece (a piece = the part of the range inside one segment) and
// atomicMax-es the float bit pattern (order-preserving for values >= 0,
// hence exact and deterministic) into ws[seg].  The last CTA to finish
// (ticket counter at ws[nseg]) turns the maxima into the outputs, then
// resets ws to zero for the next call.
template <class SEG, bool U = false>
__global__ void __launch_bounds__(kThreads) k_amax(const uint4* __restrict__ x, int64_t nblocks,
                                                   SEG seg, uint32_t* ws, float* s_t_out,
                                                   float* amax_out, int32_t* status) {
  pdl_enter();
  __shared__ uint32_t red[kThreads / 32];
  __shared__ int last;
  const int64_t b0 = cta_begin(blockIdx.x, gridDim.x, nblocks);
  const int64_t b1 = cta_begin(blockIdx.x + 1, gridDim.x, nblocks);
  const int tid = threadIdx.x;
  int64_t lo = b0;
  while (lo < b1) {
    const int s = seg.find(lo);
    const int64_t hi = (s + 1 < seg.count()) ? min(b1, seg.start(s + 1)) : b1;
    const uint4* xs = seg.xptr(s, x);
    // chunks [2lo, 2hi), 8 in flight per thread
    const int64_t c0 = 2 * lo, c1 = 2 * hi;
    uint32_t m = 0;
    int64_t c = c0 + tid;
    for (; c + 7 * kThreads < c1; c += 8 * kThreads) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = unit_ok(c + u * kThreads, c0, c1, 2 * nblocks) ? __ldg(xs + c + u * kThreads) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m = vmax_u16x2(m, v[u].x & 0x7FFF7FFFu);
        m = vmax_u16x2(m, v[u].y & 0x7FFF7FFFu);
        m = vmax_u16x2(m, v[u].z & 0x7FFF7FFFu);
        m = vmax_u16x2(m, v[u].w & 0x7FFF7FFFu);
      }
    }
    for (; c < c1; c += kThreads) {
      const uint4 v = unit_ok(c, c0, c1, 2 * nblocks) ? __ldg(xs + c) : make_uint4(0u, 0u, 0u, 0u);
      m = vmax_u16x2(m, v.x & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v.y & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v.z & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v.w & 0x7FFF7FFFu);
    }
    uint32_t mb = max(m & 0xFFFFu, m >> 16);
    mb = __reduce_max_sync(0xFFFFFFFFu, mb);
    if ((tid & 31) == 0) red[tid >> 5] = mb;
    __syncthreads();
    if (tid == 0) {
      uint32_t t = red[0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) t = max(t, red[w]);
      if (unit_ok(s, 0, seg.count(), seg.count())) atomicMax(ws + s, t << 16);
    }
    __syncthreads();
    lo = hi;
  }
  // completion ticket
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(ws + seg.count(), 1u);
    last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int k = tid; k < seg.count(); k += kThreads) {
    const uint32_t bits = atomicExch(ws + k, 0u);
    const float amax = __uint_as_float(bits);
    if (amax_out) {
      amax_out[k] = amax;
      if (!(amax <= 3.4028234663852886e38f) && status) atomicOr(status, TF4_DEV_NONFINITE);
    }
    if (s_t_out) s_t_out[k] = tensor_scale<U>(amax, status);
  }
  if (tid == 0) ws[seg.count()] = 0u;
}

// ------------------------------------------------ per-segment scale tables
// Within one segment (tensor scale s_t) an NVFP4 block with E4M3 scale code
// b = (e_b, m_b), e_b >= 1, has S = fl(s_t * (1 + m_b/8) * 2^(e_b-7))
// = S_c[m_b] * 2^(e_b-7) with S_c[m] = fl(s_t * (1 + m/8)) (power-of-two
// scaling commutes with rounding in the normal range).  So a segment has
// only 8 scale classes, and a few per-class constants replace the per-block
// divisions:
//  * rho[c]: a multiplier near 1/S_c such that, for every bf16 value v,
//    RN(v * rho) lies on the same side of every decision point (E2M1
//    midpoints for round-to-nearest, codewords for guided rounding) as the
//    exact quotient v / S_c, and equals a decision point exactly iff v / S_c
//    does.  Only the bf16 values next to a point * S_c can break this (all
//    others are >= 2^-8 away, relative, while rho's error is < 2^-20), so
//    each candidate (RN(1/S_c) +- up to 4 ulps) is checked on exactly those
//    values with an exact FMA test; rho = 0 marks a class for which no
//    candidate works (its blocks take the exact per-element path).
//  * code[m]: the E4M3 scale code of bamax = (1 + m/128) * 2^(E0-127); for
//    bamax = that * 2^k the code is code[m] + 8k while it stays a normal,
//    unsaturated E4M3 value (both roundings are scale-invariant there).
struct SegTables {
  float rho[8];
  uint32_t mask[8];  // candidate pass bits: [0, 9) round-to-nearest, [9, 18) toward zero
  int E0;
  int fast;
  int rz;            // 1: the multiplies round toward zero (chosen per segment)
  uint8_t code[128];
};

constexpr int kCand = 9;
// candidate k -> ulp offset 0, +1, -1, +2, -2, ...
__device__ __forceinline__ int cand_offset(int k) { return (k & 1) ? ((k + 1) >> 1) : -(k >> 1); }

// Decision points: the grid's midpoints (i = 0..6, tie -> upper iff i odd)
// or its nonzero codewords (i = 0..6 -> V[i+1]).
template <bool U, bool MIDPOINTS>
__device__ __forceinline__ float decision_point(int i) {
  return MIDPOINTS ? grid_mid<U>(i) : grid_value<U>((uint32_t)i + 1u);
}

template <bool RZ>
__device__ __forceinline__ float mul(float a, float b) {
  return RZ ? __fmul_rz(a, b) : __fmul_rn(a, b);
}

// All threads of the CTA call this (it synchronizes).  The multiplies may
// round to nearest or toward zero (both are odd functions, so signed inputs
// keep their symmetry); one mode is chosen per segment so that the block
// loop stays uniform: toward zero if every class has a safe multiplier in
// that mode, else to nearest if every class has one there, else the mode
// with more safe classes (the others take the exact path).
template <bool U, bool MIDPOINTS, bool CODE_TABLE = MIDPOINTS>
__device__ void build_tables(float st, SegTables& t) {
  const int tid = threadIdx.x;
  __syncthreads();  // the previous piece is done with t
  const bool fast = st >= 0x1p-90f && st <= 0x1p100f;
  if (tid < 8) t.mask[tid] = (1u << (2 * kCand)) - 1u;
  if (CODE_TABLE) {
    const int E0 = fast ? (int)((__float_as_uint(__fmul_rn(st, 448.0f * kGridMax<U>)) >> 23) & 0xFFu) - 2 : 0;
    if (tid == 0) {
      t.E0 = E0;
      t.fast = fast && E0 >= 4;
    }
    if (fast && E0 >= 4 && tid < 128) {
      const float bam = __uint_as_float(((uint32_t)E0 << 23) | ((uint32_t)tid << 16));
      t.code[tid] = (uint8_t)e4m3_encode(__fdiv_rn(__fdiv_rn(bam, kGridMax<U>), st));
    }
  } else if (tid == 0) {
    t.fast = fast;
  }
  __syncthreads();
  if (fast && tid < 8 * 28) {
    const int c = tid / 28, r = tid % 28, i = r >> 2, o = (r & 3) - 1;
    const float Sc = __fmul_rn(st, 1.0f + 0.125f * (float)c);
    const float pt = decision_point<U, MIDPOINTS>(i);
    const float P = __fmul_rn(pt, Sc);
    const float v = __uint_as_float((uint32_t)((int)(__float_as_uint(P) >> 16) + o) << 16);
    const float e = fmaf(-pt, Sc, v);  // exact sign: Sc >= 2^-96
    const uint32_t r0 = __float_as_uint(__frcp_rn(Sc));
    const bool up = (i & 1) != 0;
    uint32_t pass = 0;
#pragma unroll
    for (int k = 0; k < 2 * kCand; ++k) {
      const float rk = __uint_as_float(r0 + cand_offset(k % kCand));
      const float p = k < kCand ? __fmul_rn(v, rk) : __fmul_rz(v, rk);
      bool ok;
      if (MIDPOINTS) ok = ((e > 0.0f) || (e == 0.0f && up)) == ((p > pt) || (p == pt && up));
      else ok = ((e > 0.0f) == (p > pt)) && ((e == 0.0f) == (p == pt));
      pass |= (ok ? 1u : 0u) << k;
    }
    atomicAnd(&t.mask[c], pass);
  }
  __syncthreads();
  if (tid < 32) {
    const uint32_t m = tid < 8 ? t.mask[tid] : 0u;
    const uint32_t lane = tid < 8 ? 0xFFu : 0u;
    const uint32_t rz_ok = __ballot_sync(0xFFFFFFFFu, (m >> kCand) != 0u) & lane;
    const uint32_t rn_ok = __ballot_sync(0xFFFFFFFFu, (m & ((1u << kCand) - 1u)) != 0u) & lane;
    const bool rz = rz_ok == 0xFFu ? true : rn_ok == 0xFFu ? false : __popc(rz_ok) >= __popc(rn_ok);
    if (tid < 8) {
      const uint32_t mm = rz ? (m >> kCand) : (m & ((1u << kCand) - 1u));
      float rho = 0.0f;
      if (fast && mm) {
        const float Sc = __fmul_rn(st, 1.0f + 0.125f * (float)tid);
        rho = __uint_as_float(__float_as_uint(__frcp_rn(Sc)) + cand_offset(__ffs(mm) - 1));
      }
      t.rho[tid] = rho;
    }
    if (tid == 0) t.rz = rz;
  }
  __syncthreads();
}

// rho of class m_b scaled by 2^(7 - e_b) (exact exponent shift).
__device__ __forceinline__ float block_rho(float rho_c, uint32_t e_b) {
  return __uint_as_float(__float_as_uint(rho_c) + (uint32_t)((7 - (int)e_b) << 23));
}

// Uniform grid through the E2M3 conversion: the E2M3 values below 2 are
// the multiples of 1/8 (subnormals m/8, then 1 + m/8), so for |v| < 7.5 RNE
// of v/8 to E2M3 is RNE of v to an integer k <= 7, held in the code's
// magnitude bits (ties to even m are ties to even k); v/8 = RN(x r)/8 =
// RN(x (r/8)) exactly (a power-of-two factor; below the normal range both
// round to code 0).  CLAMP: larger |v| (magnitude bits >= 8, up to the
// satfinite maximum) saturate to k = 7.  Byte s << 5 | k -> nibble
// s << 3 | k.  (Non-finite inputs give unspecified codes.)
template <bool RZ, bool CLAMP>
__device__ __forceinline__ uint32_t cvt_uni_words(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r) {
  const float r8 = r * 0.125f;
  uint32_t b[2];  // E2M3 bytes of the even / odd elements (element 2j, 2j + 1 in byte j)
  cvt_e2m3x8(mul<RZ>(bf_lo(w0), r8), mul<RZ>(bf_lo(w1), r8), mul<RZ>(bf_lo(w2), r8), mul<RZ>(bf_lo(w3), r8),
             mul<RZ>(bf_hi(w0), r8), mul<RZ>(bf_hi(w1), r8), mul<RZ>(bf_hi(w2), r8), mul<RZ>(bf_hi(w3), r8), b[0],
             b[1]);
  if (CLAMP && ((b[0] | b[1]) & 0x18181818u)) {  // some magnitude >= 8 (rare unless train values leave the grid)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t t = (b[h] | (b[h] >> 1)) & 0x08080808u;  // magnitude >= 8
      b[h] |= t - (t >> 3);                                   // -> low three bits all ones
    }
  }
  // even element -> low nibble of byte j, odd -> high nibble: s << 3 | k
  return ((b[0] >> 2) & 0x08080808u) | (b[0] & 0x07070707u) | ((b[1] << 2) & 0x80808080u) |
         ((b[1] << 4) & 0x70707070u);
}

// Eight bf16 (four words) times rho -> eight grid nibbles (signed, RNE).
// CLAMP (uniform grid only; E2M1's conversion always saturates): the
// products may reach 7.5 or more.
template <bool RZ = false, bool U = false, bool CLAMP = true>
__device__ __forceinline__ uint32_t cvt_words(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r) {
  if constexpr (U) return cvt_uni_words<RZ, CLAMP>(w0, w1, w2, w3, r);
  return cvt_e2m1x8(mul<RZ>(bf_lo(w0), r), mul<RZ>(bf_hi(w0), r), mul<RZ>(bf_lo(w1), r),
                    mul<RZ>(bf_hi(w1), r), mul<RZ>(bf_lo(w2), r), mul<RZ>(bf_hi(w2), r),
                    mul<RZ>(bf_lo(w3), r), mul<RZ>(bf_hi(w3), r));
}

// --------------------------------------------------------- quantize pass
enum { kRTN = 0, kSR = 1, kCAPTURE = 2 };

// Philox key schedule of the SR seed (philox_schedule), a kernel parameter
// of its own: inside QuantArgs it raised every quantize variant's register
// count (48 -> 57-64 for RTN/capture), costing a resident CTA per SM.
struct PhiloxKeys {
  uint32_t ks[kPhiloxKeys];
};

struct QuantArgs {
  const uint4* x;
  int64_t nblocks;
  const float* st_src;  // s_t per segment, or amax per segment (st_from_amax)
  int st_from_amax;
  float* s_t_out;       // written by CTA 0 when st_from_amax
  uint8_t* codes;
  uint8_t* scales;
  uint8_t* bits;        // capture only; may be NULL
  uint64_t seed;
  int32_t* status;
};

// One block of an E4M3-scaled format (16 bf16 in w[0..7]; E2M1 grid for
// NVFP4, uniform grid if U) -> code words, scale byte, flags.
template <bool U, int MODE, bool RZ>
__device__ __forceinline__ void nvfp4_block(const uint32_t (&w)[8], float st, const SegTables& t,
                                            int64_t blk, const uint32_t* ks, uint32_t& c0, uint32_t& c1,
                                            uint32_t& sc, bool& bad) {
  const uint32_t mb = block_absmax_bits(w);
  bad = mb >= 0x7F80u;
  if (t.fast && !bad) {
    const int E = (int)(mb >> 7);
    const int code = (int)t.code[mb & 0x7Fu] + 8 * (E - t.E0);
    if (E >= 4 && code >= 8) {
      sc = (uint32_t)min(code, 0x7E);
      const float rho = t.rho[sc & 7u];
      if (rho != 0.0f) {
        const float r = block_rho(rho, sc >> 3);
        if (MODE != kSR) {
          // normal E4M3 scale: y <= 7 (1 + 1/16) (1 + 2^-20) < 7.5, no clamp
          c0 = cvt_words<RZ, U, false>(w[0], w[1], w[2], w[3], r);
          c1 = cvt_words<RZ, U, false>(w[4], w[5], w[6], w[7], r);
          return;
        } else {
          // stochastic rounding on the codeword-safe product; rare
          // ambiguous thresholds are decided exactly
          const float S = __fmul_rn(st, e4m3_decode(sc));
          const PhiloxBlk pb = philox_block((uint64_t)blk * 16u, ks);
          const uint32_t lo32 = (uint32_t)((uint64_t)blk * 16u);
          if constexpr (!U) {
            const float r2 = __uint_as_float(__float_as_uint(r) + 0x00800000u);  // 2 rho, exact
            uint32_t c[2] = {0u, 0u};
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const uint32_t h = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xFFFFu);
              const float ax = __uint_as_float((h & 0x7FFFu) << 16);
              const uint32_t pw = philox_w0_blk(lo32 + (uint32_t)k, pb, ks);
              bool amb;
              uint32_t m3 = sr_e2m1(mul<RZ>(ax, r2), pw, amb);
              if (amb) m3 = sr_m3_exact<false>(ax, S, pw >> 8);
              c[k >> 3] |= (m3 | ((h >> 12) & 8u)) << (4 * (k & 7));
            }
            c0 = c[0];
            c1 = c[1];
          } else {
            uint32_t c[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {  // 8 elements at a time
              float v[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int k = 8 * q + e;
                const uint32_t h = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xFFFFu);
                const float ax = __uint_as_float((h & 0x7FFFu) << 16);
                const uint32_t r24 = philox_w0_blk(lo32 + (uint32_t)k, pb, ks) >> 8;
                bool amb;
                float val = sr_pick_uni(mul<RZ>(ax, r), r24, amb);
                if (amb) val = grid_value<U>(sr_m3_exact<U>(ax, S, r24));
                v[e] = __uint_as_float(__float_as_uint(val) | ((h & 0x8000u) << 16));
              }
              c[q] = cvt_grid_x8<U>(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
            }
            c0 = c[0];
            c1 = c[1];
          }
          return;
        }
      }
    }
  }
  // Exact path: scale by the defining divisions, decisions by exact
  // comparisons (E4M3-subnormal or zero scales, classes without a safe
  // multiplier, tiny segments).
  float S = 0.0f;
  sc = 0;
  if (st > 0.0f) {  // st == 0: zero segment; NaN: non-finite segment
    const float bamax = __uint_as_float(mb << 16);
    sc = e4m3_encode(__fdiv_rn(__fdiv_rn(bamax, kGridMax<U>), st));
    S = __fmul_rn(st, e4m3_decode(sc));
  }
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t h = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xFFFFu);
    const float ax = __uint_as_float((h & 0x7FFFu) << 16);
    uint32_t m3 = 0;
    if (S > 0.0f) {
      if constexpr (MODE == kSR)
        m3 = sr_m3_exact<U>(ax, S, philox_w0_blk((uint32_t)((uint64_t)blk * 16u) + (uint32_t)k,
                                                 philox_block((uint64_t)blk * 16u, ks), ks) >> 8);
      else
        m3 = rtn_m3_exact<U>(ax, S);
    }
    out[k >> 3] |= (((h >> 15) << 3) | m3) << (4 * (k & 7));
  }
  c0 = out[0];
  c1 = out[1];
}

// MXFP4 stochastic rounding where y = |x| 2^-e underflowed to 0 for a
// nonzero x (possible only for e > 16): the exact threshold is then in
// (0, 1), so the element rounds up to 0.5 iff r24 == 0 (rare; kept out of
// the main loop's registers).
__device__ __noinline__ void mxfp4_sr_underflow(const uint32_t (&w)[16], float inv, uint32_t lo32,
                                               const PhiloxBlk& pb, const uint32_t* ks, uint32_t (&c)[4]) {
#pragma unroll 1
  for (int k = 0; k < 32; ++k) {
    const uint32_t h = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xFFFFu);
    const float ax = __uint_as_float((h & 0x7FFFu) << 16);
    if (ax != 0.0f && __fmul_rn(ax, inv) == 0.0f && (philox_w0_blk(lo32 + (uint32_t)k, pb, ks) >> 8) == 0u)
      c[k >> 3] |= 1u << (4 * (k & 7));  // m3 0 -> 1, the sign nibble bit kept
  }
}

// One MXFP4 block (32 bf16 in w[0..15]) -> code words, scale byte, flags.
template <int MODE>
__device__ __forceinline__ void mxfp4_block(const uint32_t (&w)[16], int64_t blk, const uint32_t* ks,
                                            uint32_t (&c)[4], uint32_t& sc, bool& bad) {
  const uint32_t mb = block_absmax_bits(w);
  bad = mb >= 0x7F80u;
  const uint32_t E = (mb >> 7) & 0xFFu;  // bf16 exponent field of bamax
  // e = floor(log2 bamax) - 2 clamped at -127; bamax subnormal or 0 -> -127
  const int e = (E == 0) ? -127 : max((int)E - 129, -127);
  sc = (uint32_t)(e + 127);
  if (MODE != kSR) {
    // y = x * 2^-e is exact (2^-e is a normal fp32 for e in [-127, 125]),
    // so hardware RNE of y is the exact answer.
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
#pragma unroll
    for (int q = 0; q < 4; ++q) c[q] = cvt_words(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3], inv);
    return;
  }
  // stochastic rounding on the quotient y = |x| * 2^-e, exact unless it
  // underflows (possible only for e > 16: |x| >= 2^-133); a nonzero x whose
  // y underflows to 0 has 0 < 2^24 (y - lo) / gap < 1, so it rounds up
  // exactly when r24 == 0
  const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
  const PhiloxBlk pb = philox_block((uint64_t)blk * 32u, ks);
  const uint32_t lo32 = (uint32_t)((uint64_t)blk * 32u);
  float v[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const uint32_t h = (k & 1) ? (w[k >> 1] >> 16) : (w[k >> 1] & 0xFFFFu);
    const float ax = __uint_as_float((h & 0x7FFFu) << 16);
    const float val = sr_pick_e2m1_exact(__fmul_rn(ax, inv), philox_w0_blk(lo32 + (uint32_t)k, pb, ks) >> 8);
    v[k] = __uint_as_float(__float_as_uint(val) | ((h & 0x8000u) << 16));
  }
#pragma unroll
  for (int q = 0; q < 4; ++q)
    c[q] = cvt_e2m1x8(v[8 * q], v[8 * q + 1], v[8 * q + 2], v[8 * q + 3], v[8 * q + 4], v[8 * q + 5],
                      v[8 * q + 6], v[8 * q + 7]);
  if (e > 16) mxfp4_sr_underflow(w, inv, lo32, pb, ks, c);
}

// A hint that brings the line holding p into L2 (no data returned, no
// fault semantics beyond those of a load; every caller passes an address
// inside the buffer it is about to read).
__device__ __forceinline__ void l2_prefetch(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ void report_bad(bool bad, int32_t* status) {
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0 && status)
    atomicOr(status, TF4_DEV_NONFINITE);
}

// Quantize pass.  CTAs take the amax pass's ranges in reverse order (CTA i
// gets range G-1-i) and walk them backwards, so that the first blocks read
// are the ones the amax pass read last (still in L2).  Each lane also asks
// L2 for its input of the next iteration (one `prefetch.global.L2` per
// block): the walk runs towards lower addresses, and the explicit request
// keeps the backward stream's DRAM reads ahead of the loads.
// Resident CTAs per SM asked of the compiler (0: its own choice).  The
// ragged-segment nearest / capture variants are held to 5 (48 registers,
// a few loop invariants spilled), which measured 2-3% faster on the MoE
// dispatch workload than the 64 registers / 4 CTAs they take otherwise;
// the batched variants lost that way (MXFP4: 140 -> 175 us for 40 layers
// of 4096x2048), and a bound of 1 lets the compiler take far more
// registers, so every other variant keeps the compiler's choice.
template <int MODE, class SEG>
constexpr int quant_min_ctas() {
  return (MODE != kSR && std::is_same<SEG, SegN>::value) ? 5 : 0;
}

// The quantize pass over the CTA's block range [b0, b1), walked backwards
// (shared by the two-launch and the single-launch capture).
// `stage` (may be NULL): the CTA's blocks [b0, b1) already in shared memory
// (16-element formats only), read from there instead of from x.
template <int FMT, int MODE, class SEG>
__device__ __forceinline__ void quant_range(const QuantArgs& a, const SEG& seg, const PhiloxKeys& pk, SegTables& tb,
                                            int64_t b0, int64_t b1, const uint4* stage = nullptr) {
  // blocks per lane per iteration: 2 keeps 64 B per lane in flight for the
  // memory-bound modes; stochastic rounding is bound by the integer pipe
  // and gains more from the registers (resident warps) one block saves
  constexpr int U = MODE == kSR ? 1 : 2;
  const int tid = threadIdx.x;
  constexpr bool UG = kUni<FMT>;
  if (kE4M3<FMT> && a.st_from_amax && blockIdx.x == 0 && a.s_t_out)
    for (int k = tid; k < seg.count(); k += kThreads) a.s_t_out[k] = tensor_scale<UG>(a.st_src[k], a.status);
  int64_t hi = b1;
  while (hi > b0) {
    const int s = seg.find(hi - 1);
    const int64_t lo = max(b0, seg.start(s));
    float st = 0.0f;
    if constexpr (kE4M3<FMT>) {
      st = a.st_from_amax ? tensor_scale<UG>(a.st_src[s], nullptr) : a.st_src[s];
      if (MODE != kSR) build_tables<UG, true>(st, tb);
      else build_tables<UG, false, true>(st, tb);
    }
    const uint4* xs = seg.xptr(s, a.x);
    uint8_t* bits = seg.bitsptr(s, a.bits);
    const int64_t n = hi - lo;
    for (int64_t j = 0; j < n; j += (int64_t)U * kThreads) {
      if constexpr (kE4M3<FMT>) {
        uint32_t w[U][8];
        int64_t blk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t k = j + u * kThreads + tid;
          blk[u] = hi - 1 - k;
          if (!stage && k + (int64_t)U * kThreads < n && unit_ok(blk[u] - (int64_t)U * kThreads, lo, hi, a.nblocks))
            l2_prefetch(xs + 2 * (blk[u] - (int64_t)U * kThreads));
          if (k < n && unit_ok(blk[u], lo, hi, a.nblocks)) {
            uint4 p, q;
            if (stage) {
              p = stage[2 * (blk[u] - b0)];
              q = stage[2 * (blk[u] - b0) + 1];
            } else {
              p = __ldg(xs + 2 * blk[u]);
              q = __ldg(xs + 2 * blk[u] + 1);
            }
            w[u][0] = p.x; w[u][1] = p.y; w[u][2] = p.z; w[u][3] = p.w;
            w[u][4] = q.x; w[u][5] = q.y; w[u][6] = q.z; w[u][7] = q.w;
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const bool valid = j + u * kThreads + tid < n;
          bool bad = false;
          if (valid && unit_ok(blk[u], lo, hi, a.nblocks)) {
            uint32_t c0, c1, sc;
            if (tb.rz)
              nvfp4_block<UG, MODE, true>(w[u], st, tb, blk[u], pk.ks, c0, c1, sc, bad);
            else
              nvfp4_block<UG, MODE, false>(w[u], st, tb, blk[u], pk.ks, c0, c1, sc, bad);
            reinterpret_cast<uint2*>(a.codes)[blk[u]] = make_uint2(c0, c1);
            a.scales[blk[u]] = (uint8_t)sc;
            if (MODE == kCAPTURE && bits)
              reinterpret_cast<uint16_t*>(bits)[blk[u]] =
                  (uint16_t)(nibble_lsbs(c0) | (nibble_lsbs(c1) << 8));
          }
          report_bad(bad, a.status);
        }
      } else {
        uint32_t w[U][16];
        int64_t blk[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t k = j + u * kThreads + tid;
          blk[u] = hi - 1 - k;
          if (k + (int64_t)U * kThreads < n && unit_ok(blk[u] - (int64_t)U * kThreads, lo, hi, a.nblocks))
            l2_prefetch(xs + 4 * (blk[u] - (int64_t)U * kThreads));
          if (k < n && unit_ok(blk[u], lo, hi, a.nblocks)) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 p = __ldg(xs + 4 * blk[u] + q);
              w[u][4 * q] = p.x; w[u][4 * q + 1] = p.y; w[u][4 * q + 2] = p.z; w[u][4 * q + 3] = p.w;
            }
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const bool valid = j + u * kThreads + tid < n;
          bool bad = false;
          if (valid && unit_ok(blk[u], lo, hi, a.nblocks)) {
            uint32_t c[4], sc;
            mxfp4_block<MODE>(w[u], blk[u], pk.ks, c, sc, bad);
            reinterpret_cast<uint4*>(a.codes)[blk[u]] = make_uint4(c[0], c[1], c[2], c[3]);
            a.scales[blk[u]] = (uint8_t)sc;
            if (MODE == kCAPTURE && bits)
              reinterpret_cast<uint32_t*>(bits)[blk[u]] =
                  nibble_lsbs(c[0]) | (nibble_lsbs(c[1]) << 8) | (nibble_lsbs(c[2]) << 16) |
                  (nibble_lsbs(c[3]) << 24);
          }
          report_bad(bad, a.status);
        }
      }
    }
    hi = lo;
  }
}

template <int FMT, int MODE, class SEG>
__global__ void __launch_bounds__(kThreads, quant_min_ctas<MODE, SEG>()) k_quant(QuantArgs a, SEG seg, PhiloxKeys pk) {
  pdl_enter();
  __shared__ SegTables tb;
  const int64_t ci = (int64_t)gridDim.x - 1 - blockIdx.x;
  quant_range<FMT, MODE, SEG>(a, seg, pk, tb, cta_begin(ci, gridDim.x, a.nblocks),
                              cta_begin(ci + 1, gridDim.x, a.nblocks));
}

// ------------------------------------------- single-launch capture (small)
// The amax pass and the quantize pass of an NVFP4 / UFP4 tensor with one
// segment in one cooperative launch (all CTAs resident at once): each CTA
// reduces max |x| over its block range and atomicMax-es it into ws[0], then
// counts itself in ws[1]; thread 0 waits until all gridDim.x CTAs have
// arrived, and the CTA quantizes the same range, backwards, which it read
// just before (for a tensor that fits in L2, from L2).  The wait is bounded
// by wait_ns of %globaltimer: a CTA that gives up ORs TF4_DEV_TIMEOUT into
// the status word and returns (its outputs are then unspecified, and ws is
// left as it is).  The last CTA to finish (ws[2]) zeroes ws[0..2].
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// STAGED: the CTA's 16-byte chunks read by the amax phase are also kept in
// dynamic shared memory (the host sizes it to the largest range), and the
// quantize phase reads them from there.
template <int FMT, int MODE, bool STAGED>
__global__ void __launch_bounds__(kThreads) k_quant_fused(QuantArgs a, uint32_t* ws, PhiloxKeys pk,
                                                          uint64_t wait_ns) {
  extern __shared__ uint4 stage[];
  __shared__ SegTables tb;
  __shared__ uint32_t red[kThreads / 32];
  __shared__ float amax_sh;
  __shared__ int arrived;
  const int64_t b0 = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
  const int64_t b1 = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  const int tid = threadIdx.x;
  // phase 1: max |x| over the range, 16-byte chunks, 8 in flight per thread
  const int64_t c0 = 2 * b0, c1 = 2 * b1;
  uint32_t m = 0;
  int64_t c = c0 + tid;
  for (; c + 7 * kThreads < c1; c += 8 * kThreads) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      v[u] = unit_ok(c + u * kThreads, c0, c1, 2 * a.nblocks) ? __ldg(a.x + c + u * kThreads) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (STAGED) stage[c + u * kThreads - c0] = v[u];
      m = vmax_u16x2(m, v[u].x & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v[u].y & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v[u].z & 0x7FFF7FFFu);
      m = vmax_u16x2(m, v[u].w & 0x7FFF7FFFu);
    }
  }
  for (; c < c1; c += kThreads) {
    const uint4 v = unit_ok(c, c0, c1, 2 * a.nblocks) ? __ldg(a.x + c) : make_uint4(0u, 0u, 0u, 0u);
    if (STAGED) stage[c - c0] = v;
    m = vmax_u16x2(m, v.x & 0x7FFF7FFFu);
    m = vmax_u16x2(m, v.y & 0x7FFF7FFFu);
    m = vmax_u16x2(m, v.z & 0x7FFF7FFFu);
    m = vmax_u16x2(m, v.w & 0x7FFF7FFFu);
  }
  uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, max(m & 0xFFFFu, m >> 16));
  if ((tid & 31) == 0) red[tid >> 5] = mb;
  __syncthreads();
  if (tid == 0) {
    uint32_t t = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) t = max(t, red[w]);
    atomicMax(ws, t << 16);
    __threadfence();
    atomicAdd(ws + 1, 1u);
    // grid-wide wait for every CTA's maximum, bounded
    const uint64_t t0 = global_ns();
    int ok = 1;
    while (ld_acquire(ws + 1) != gridDim.x) {
      if (global_ns() - t0 > wait_ns) {
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    arrived = ok;
    if (ok) amax_sh = __uint_as_float(__ldcg(ws));
  }
  __syncthreads();
  if (!arrived) {
    if (tid == 0 && a.status) atomicOr(a.status, TF4_DEV_TIMEOUT);
    return;
  }
  // phase 2: the quantize pass with the tensor amax
  QuantArgs q = a;
  q.st_src = &amax_sh;
  q.st_from_amax = 1;
  quant_range<FMT, MODE, Seg1>(q, Seg1{}, pk, tb, b0, b1, STAGED ? stage : nullptr);
  // the last CTA out returns the workspace to zero
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(ws + 2, 1u) == gridDim.x - 1) {
      ws[0] = 0u;
      ws[1] = 0u;
      ws[2] = 0u;
    }
  }
}

// ----------------------------------------------------------- guided pass
// Guided rounding picks, of the two codewords lo <= y < hi around y, the
// one whose m3 & 1 equals the recorded bit (y a codeword keeps itself;
// y >= grid max gives 7).  With the floor code f of y and y strictly
// between codewords, that is f + ((f ^ g) & 1): only the floor and whether
// y sits exactly on a codeword are needed, never the nearest code.
//
// Both come, for eight elements at once, from one rounding of y to a grid
// four times finer whose points include every codeword: E2M3 (2 exponent
// bits, 3 mantissa bits, subnormals 0..7/8) for the E2M1 grid -- an E2M1
// value with code m3 is the E2M3 value with code m3 << 2 -- and the
// half-integers for the uniform grid.  Let N be the fine code of y
// (hardware RNE; for the uniform grid the E2M3 rounding of y/4, whose
// spacing below 2 is 1/8, i.e. y to a multiple of 1/2), f = N >> 2 its
// codeword part and l = N & 3 the rest (uniform grid: N = 2f + l, l = N & 1):
//  * l != 0: N lies strictly between two codewords, and so does y (a tie
//    between N and a codeword goes to the codeword, whose code is even):
//    the answer is f + ((f ^ g) & 1), capped at 7;
//  * l == 0: y lies within half a fine step of the codeword c = f, hence
//    strictly between c's two neighbours.  If c's bit equals g the answer
//    is c wherever y is; otherwise it is c - 1, c or c + 1 by the side of c
//    that y is on, decided element by element (rare: it needs a train
//    value next to a codeword the rollout did not choose).
// With a codeword-safe product y (it is on the same side of every nonzero
// codeword as the exact quotient, and equal to one iff the quotient is),
// every step above holds for the exact quotient too; zero is decided on
// the bf16 value itself, since a nonzero x times r may underflow to 0.
// The fine codes are handled four to a 32-bit word, one per byte laid out
// as s << 5 | f << 2 | l.
struct GuidedArgs {
  const uint4* x;
  int64_t nblocks;
  const uint8_t* rec_scales;
  const float* rec_s_t;
  const uint8_t* rec_bits;
  uint8_t* codes;
  int32_t* status;
};

// Fine codes of eight elements (bf16 pairs w0..w3) times r, one byte each
// as above: b0 holds the even elements (element 2j in byte j), b1 the odd
// ones (element 2j + 1 in byte j), so that one shift-and-merge puts both
// into nibble order.  Uniform grid: N = RN(2 min(|y|, 7.5)), from RNE of
// y/4 to E2M3 (as in cvt_uni_words, at half the step): byte s << 5 | N,
// N clamped to 15 when CLAMP.
template <bool RZ, bool U, bool CLAMP>
__device__ __forceinline__ void fine_codes(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r,
                                           uint32_t& b0, uint32_t& b1) {
  const float rr = U ? r * 0.25f : r;
  cvt_e2m3x8(mul<RZ>(bf_lo(w0), rr), mul<RZ>(bf_lo(w1), rr), mul<RZ>(bf_lo(w2), rr), mul<RZ>(bf_lo(w3), rr),
             mul<RZ>(bf_hi(w0), rr), mul<RZ>(bf_hi(w1), rr), mul<RZ>(bf_hi(w2), rr), mul<RZ>(bf_hi(w3), rr), b0, b1);
  if constexpr (U) {
    if (CLAMP && ((b0 | b1) & 0x10101010u)) {  // some N >= 16 (rare unless train values leave the grid)
      const uint32_t t0 = b0 & 0x10101010u, t1 = b1 & 0x10101010u;
      b0 |= t0 - (t0 >> 4);                    // -> low four bits all ones
      b1 |= t1 - (t1 >> 4);
    }
  }
}

// 8 guidance bits -> bit 0 of 8 nibbles (shift-or steps written as
// multiplies: the shifted copies never overlap).
__device__ __forceinline__ uint32_t spread_bits(uint32_t b) {
  uint32_t x = b & 0xFFu;
  x = (x * 0x1001u) & 0x000F000Fu;
  x = (x * 0x41u) & 0x03030303u;
  x = (x * 0x9u) & 0x11111111u;
  return x;
}

// The side test for the flagged elements (fl: bit 0 of their nibbles):
// c = f of the fine code (P's nibble, recorded bit different from c's), so
// y == c (or y >= grid max at c = 7) keeps c, otherwise the answer is the
// neighbour on y's side; zero is decided on x itself.
template <bool RZ, bool U>
__device__ __noinline__ uint32_t guided_sides(uint32_t c, uint32_t P, uint32_t fl, uint32_t w0, uint32_t w1,
                                              uint32_t w2, uint32_t w3, float r) {
  while (fl) {
    const int e = (__ffs(fl) - 1) >> 2;
    fl &= fl - 1u;
    const uint32_t f = (P >> (4 * e)) & 7u;
    const uint32_t wk = (e & 4) ? ((e & 2) ? w3 : w2) : ((e & 2) ? w1 : w0);
    const uint32_t h = (e & 1) ? (wk >> 16) : (wk & 0xFFFFu);
    const float y = mul<RZ>(__uint_as_float((h & 0x7FFFu) << 16), r);
    const float v = grid_value<U>(f);
    uint32_t m3;
    if (f == 0u) m3 = (h & 0x7FFFu) ? 1u : 0u;
    else if (y == v || (f == 7u && y >= kGridMax<U>)) m3 = f;
    else m3 = y > v ? f + 1u : f - 1u;
    c = (c & ~(7u << (4 * e))) | (m3 << (4 * e));
  }
  return c;
}

// Guided rounding of eight elements (bf16 pairs w0..w3; recorded bits gs,
// element k's bit at bit 4k) on the codeword-safe multiplier r -> eight
// nibbles.  In nibble form (P: s << 3 | f per element) the answer is
// f + ((f ^ g) & 1) with f = 7 left as it is; elements with l = 0 whose f's
// bit differs from g take the side test.
template <bool RZ, bool U, bool CLAMP>
__device__ __forceinline__ uint32_t guided_x8_spread(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r,
                                                     uint32_t gs) {
  uint32_t be, bo;  // fine codes of the even / odd elements
  fine_codes<RZ, U, CLAMP>(w0, w1, w2, w3, r, be, bo);
  uint32_t P, L;    // s << 3 | f and (bit 0) l != 0, nibble k = element k
  if constexpr (U) {  // byte s << 5 | N, N = 2f + l
    P = ((be >> 2) & 0x08080808u) | ((be >> 1) & 0x07070707u) | ((bo << 2) & 0x80808080u) |
        ((bo << 3) & 0x70707070u);
    L = (be & 0x01010101u) | ((bo << 4) & 0x10101010u);
  } else {            // byte s << 5 | f << 2 | l
    P = ((be >> 2) & 0x0F0F0F0Fu) | ((bo << 2) & 0xF0F0F0F0u);
    L = ((be | (be >> 1)) & 0x01010101u) | (((bo | (bo >> 1)) << 4) & 0x10101010u);
  }
  const uint32_t A = (P ^ gs) & 0x11111111u;                     // f's bit != g
  const uint32_t F7 = P & (P >> 1) & (P >> 2) & 0x11111111u;    // f == 7
  const uint32_t c = P + (A & ~F7);
  const uint32_t fl = A & ~L;
  return fl ? guided_sides<RZ, U>(c, P, fl, w0, w1, w2, w3, r) : c;
}

// The same with the recorded bits g8 packed (element k in bit k).
template <bool RZ, bool U, bool CLAMP>
__device__ __forceinline__ uint32_t guided_x8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r,
                                              uint32_t g8) {
  return guided_x8_spread<RZ, U, CLAMP>(w0, w1, w2, w3, r, spread_bits(g8));
}

// The same as a call: the nearest-rounding loops recompute a word with it
// only where a lane's nearest code has the wrong bit, which keeps the fine
// rounding's registers out of their (two-unit) iteration.
template <bool RZ, bool U>
__device__ __noinline__ uint32_t guided_x8_call(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r,
                                                uint32_t g8) {
  return guided_x8<RZ, U, true>(w0, w1, w2, w3, r, g8);
}

// Guided rounding of eight elements by nearest rounding first: where the
// nearest code already carries the recorded bit it is the answer (it is one
// of y's two neighbours); `mm` gets the nibbles (bit 0) where it does not.
template <bool RZ, bool U, bool CLAMP>
__device__ __forceinline__ uint32_t nearest_x8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3, float r,
                                               uint32_t g8, uint32_t& mm) {
  const uint32_t c = cvt_words<RZ, U, CLAMP>(w0, w1, w2, w3, r);
  mm = (c ^ spread_bits(g8)) & 0x11111111u;
  return c;
}

// Per warp, guided rounding starts with nearest rounding plus the fine
// rounding for the (warp-uniform) iterations where some lane's nearest code
// has the wrong bit.  A score (one register, starting at -8) gains 4 on
// such an iteration and loses 1 on a clean one, never going below -16; once
// it passes 0 (three such iterations in a row from the start, or a run in
// which more than one iteration in five has one) the warp takes the fine
// rounding for the rest of its range.
struct GuidedMode {
  int score = -8;
  __device__ __forceinline__ bool fine() const { return score > 0; }
  // One nearest-rounding iteration; `any`: this lane needs the fine rounding.
  __device__ __forceinline__ bool note(bool any) {
    if (!__any_sync(0xFFFFFFFFu, any)) {
      score = max(score - 1, -16);
      return false;
    }
    score += 4;
    return true;
  }
};

// Per-segment tables of the guided kernels (E4M3-scaled formats), indexed
// by the recorded scale byte: the block's multiplier r (0: the block takes
// the exact comparisons) and its scale S = s_t * decode(byte), so a block
// reads both with one shared-memory load each.
struct GuidedTables : SegTables {
  float rblk[256];
  float sblk[256];
};

// After build_tables (all threads of the CTA call this; it synchronizes).
__device__ void build_block_tables(float st, GuidedTables& t) {
  static_assert(kThreads == 256, "one table entry per thread");
  const uint32_t sc = threadIdx.x;
  float r = 0.0f;
  if (t.fast && (sc >> 3) >= 1u && sc < 0x7Fu && t.rho[sc & 7u] != 0.0f) r = block_rho(t.rho[sc & 7u], sc >> 3);
  t.rblk[sc] = r;
  t.sblk[sc] = st > 0.0f ? __fmul_rn(st, e4m3_decode(sc)) : 0.0f;
  __syncthreads();
}

// Non-finite input seen by this lane (rare: each lane reports on its own,
// with no warp vote on the common path).
__device__ __forceinline__ void report_bad_lane(bool bad, int32_t* status) {
  if (bad && status) atomicOr(status, TF4_DEV_NONFINITE);
}

// One block of a guided pass: its codeword-safe multiplier r (0 when the
// block takes the exact comparisons, whose codes then go to c) and whether
// it holds a non-finite input.
template <int FMT>
__device__ __forceinline__ float guided_block_r(const uint32_t (&w)[kE4M3<FMT> ? 8 : 16], uint32_t sc, uint32_t g,
                                                const GuidedTables& tb, uint32_t (&c)[kE4M3<FMT> ? 2 : 4],
                                                bool& bad) {
  constexpr bool UG = kUni<FMT>;
  constexpr int BE = kE4M3<FMT> ? 16 : 32;
  constexpr int NQ = BE / 8;
  bad = block_absmax_bits(w) >= 0x7F80u;
  float r;
  if constexpr (kE4M3<FMT>) r = tb.rblk[sc];
  else r = (sc >= 1u && sc <= 252u) ? __uint_as_float((254u - sc) << 23) : 0.0f;  // 2^-(sc-127), exact
  if (r == 0.0f) {  // no codeword-safe multiplier: exact comparisons per element
    float S;
    if constexpr (kE4M3<FMT>) S = tb.sblk[sc];
    else S = __uint_as_float(sc >= 1u ? sc << 23 : 0x00400000u);
#pragma unroll
    for (int q = 0; q < NQ; ++q) c[q] = 0u;
#pragma unroll
    for (int e = 0; e < BE; ++e) {
      const uint32_t h = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
      const float ax = __uint_as_float((h & 0x7FFFu) << 16);
      const uint32_t m3 = S > 0.0f ? guided_m3_exact<UG>(ax, S, (g >> e) & 1u) : 0u;
      c[e >> 3] |= (((h >> 15) << 3) | m3) << (4 * (e & 7));
    }
  }
  return r;
}

template <int FMT>
__device__ __forceinline__ void guided_load(const GuidedArgs& a, int64_t blk, uint32_t (&w)[kE4M3<FMT> ? 8 : 16],
                                            uint32_t& sc, uint32_t& g) {
  constexpr int NC = kE4M3<FMT> ? 2 : 4;  // 16-B pieces of x per block
#pragma unroll
  for (int q = 0; q < NC; ++q) {
    const uint4 p = __ldg(a.x + NC * blk + q);
    w[4 * q] = p.x; w[4 * q + 1] = p.y; w[4 * q + 2] = p.z; w[4 * q + 3] = p.w;
  }
  sc = a.rec_scales[blk];
  if constexpr (kE4M3<FMT>) g = __ldg(reinterpret_cast<const uint16_t*>(a.rec_bits) + blk);
  else g = __ldg(reinterpret_cast<const uint32_t*>(a.rec_bits) + blk);
}

template <int FMT>
__device__ __forceinline__ void guided_store(const GuidedArgs& a, int64_t blk, const uint32_t (&c)[kE4M3<FMT> ? 2 : 4]) {
  if constexpr (kE4M3<FMT>) reinterpret_cast<uint2*>(a.codes)[blk] = make_uint2(c[0], c[1]);
  else reinterpret_cast<uint4*>(a.codes)[blk] = make_uint4(c[0], c[1], c[2], c[3]);
}

// One piece [lo, hi) of a CTA's range (one segment, tensor scale st, rounding
// mode of its multiplies RZ).  While the warp's mismatches are rare it runs
// nearest rounding on two blocks per lane per iteration, recomputing with
// the fine rounding (a call) only the words where some lane's nearest code
// has the wrong bit; once GuidedMode switches, the rest of the range takes
// the fine rounding, one block per lane per iteration.
template <int FMT, bool RZ>
__device__ __forceinline__ void guided_piece(const GuidedArgs& a, int64_t lo, int64_t hi,
                                             const GuidedTables& tb, GuidedMode& md) {
  constexpr bool UG = kUni<FMT>;
  constexpr int NW = kE4M3<FMT> ? 8 : 16;  // bf16 pair words per block
  constexpr int NQ = NW / 4;               // code words per block
  const int tid = threadIdx.x;
  const int64_t n = hi - lo;
  int64_t j = 0;
  for (; j < n && !md.fine(); j += 2 * kThreads) {
    uint32_t w[2][NW], sc[2], g[2];
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t k = j + u * kThreads + tid;
      ok[u] = k < n && unit_ok(lo + k, lo, hi, a.nblocks);
      if (ok[u]) guided_load<FMT>(a, lo + k, w[u], sc[u], g[u]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint32_t c[NQ], mm[NQ];
      bool bad = false;
      float r = 0.0f;
      if (ok[u]) r = guided_block_r<FMT>(w[u], sc[u], g[u], tb, c, bad);
      const bool fast = ok[u] && r != 0.0f;
      uint32_t any = 0u;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const uint32_t* wq = &w[u][4 * q];
        mm[q] = 0u;
        if (fast) c[q] = nearest_x8<RZ, UG, true>(wq[0], wq[1], wq[2], wq[3], r, g[u] >> (8 * q), mm[q]);
        any |= mm[q];
      }
      if (md.note(any != 0u)) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const uint32_t* wq = &w[u][4 * q];
          if (mm[q] != 0u) c[q] = guided_x8_call<RZ, UG>(wq[0], wq[1], wq[2], wq[3], r, g[u] >> (8 * q));
        }
      }
      if (ok[u]) guided_store<FMT>(a, lo + j + u * kThreads + tid, c);
      report_bad_lane(bad, a.status);
    }
  }
  for (; j < n; j += kThreads) {
    const int64_t k = j + tid;
    const bool ok = k < n && unit_ok(lo + k, lo, hi, a.nblocks);
    uint32_t w[NW], sc = 0u, g = 0u, c[NQ];
    bool bad = false;
    if (ok) {
      guided_load<FMT>(a, lo + k, w, sc, g);
      const float r = guided_block_r<FMT>(w, sc, g, tb, c, bad);
      if (r != 0.0f) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const uint32_t* wq = &w[4 * q];
          c[q] = guided_x8<RZ, UG, true>(wq[0], wq[1], wq[2], wq[3], r, g >> (8 * q));
        }
      }
      guided_store<FMT>(a, lo + k, c);
    }
    report_bad_lane(bad, a.status);
  }
}

// Resident CTAs per SM the guided kernels are compiled for.  They are
// latency-bound, so occupancy decides their speed more than spare
// registers: k_guided at <= 40 registers keeps 6 CTAs (48 warps) per SM for
// the 16-element formats, at <= 64 4 CTAs for MXFP4 (twice the data per
// block), k_guided_fq at <= 32 keeps 8 (64 warps).
template <int FMT>
constexpr int guided_min_ctas() {
  return kE4M3<FMT> ? 6 : 4;
}
constexpr int kGuidedFqMinCtas = 8;

template <int FMT, class SEG>
__global__ void __launch_bounds__(kThreads, guided_min_ctas<FMT>()) k_guided(GuidedArgs a, SEG seg) {
  pdl_enter();
  constexpr bool UG = kUni<FMT>;
  __shared__ GuidedTables tb;
  int s = 0;
  int64_t lo, hi;
  if constexpr (std::is_same<SEG, SegPieces>::value) {
    seg.piece(blockIdx.x, s, lo, hi);
  } else {
    lo = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
    hi = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  }
  GuidedMode md;
  if constexpr (kE4M3<FMT>) {
    const float st = a.rec_s_t[s];
    build_tables<UG, false>(st, tb);
    build_block_tables(st, tb);
  }
  if (kE4M3<FMT> && tb.rz) guided_piece<FMT, true>(a, lo, hi, tb, md);
  else guided_piece<FMT, false>(a, lo, hi, tb, md);
}

// --------------------------------------------- fused guided fake-quant
// Train-side forward in one pass: guided quantization of x against the
// rollout record, then dequantization of the chosen codes, written as fp32
// or as bf16 (round-to-nearest-even of the fp32 value), and optionally the
// codes.  Work unit = an oct of 8 consecutive elements (16 B of x in, one
// guidance byte, one code word out), so consecutive lanes read 16-B and
// write 16-B (bf16) / 2 x 16-B (fp32) pieces of one contiguous span.
struct GuidedFqArgs {
  const uint4* x;         // bf16 octs
  int64_t nblocks;
  const uint8_t* rec_scales;
  const float* rec_s_t;
  const uint8_t* rec_bits;
  uint8_t* codes;         // may be NULL
  void* out;              // 2 x float4 (fp32) or uint4 (bf16) per oct
  int32_t* status;
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Output modes of the fused pass.
enum { kOutBf16 = 0, kOutF32 = 1, kOutF32V8 = 2 };

// One oct of the fused pass: scale S of its block, codeword-safe multiplier
// r (0 when the oct takes the exact comparisons, whose codes then go to c)
// and whether it holds a non-finite input.
template <int FMT>
__device__ __forceinline__ float fq_oct_r(const uint32_t (&w)[4], uint32_t sc, uint32_t g, const GuidedTables& tb,
                                          float& S, uint32_t& c, bool& bad) {
  constexpr bool UG = kUni<FMT>;
  bad = block_absmax_bits(w) >= 0x7F80u;
  float r;
  if constexpr (kE4M3<FMT>) {
    S = tb.sblk[sc];
    r = tb.rblk[sc];
  } else {
    S = __uint_as_float(sc >= 1u ? sc << 23 : 0x00400000u);
    r = (sc >= 1u && sc <= 252u) ? __uint_as_float((254u - sc) << 23) : 0.0f;
  }
  if (r == 0.0f) {  // no codeword-safe multiplier: exact comparisons per element
    c = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t h = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
      const float ax = __uint_as_float((h & 0x7FFFu) << 16);
      const uint32_t m3 = S > 0.0f ? guided_m3_exact<UG>(ax, S, (g >> e) & 1u) : 0u;
      c |= (((h >> 15) << 3) | m3) << (4 * e);
    }
  }
  return r;
}

// Codes (optional) and dequantized values of oct o.
template <int FMT, int OUT>
__device__ __forceinline__ void fq_store(const GuidedFqArgs& a, int64_t o, uint32_t c, float S) {
  constexpr bool UG = kUni<FMT>;
  if (a.codes) reinterpret_cast<uint32_t*>(a.codes)[o] = c;
  float4 v0, v1;
  decode8_grid<UG>(c, S, v0, v1);
  if constexpr (OUT == kOutBf16) {
    reinterpret_cast<uint4*>(a.out)[o] = make_uint4(bf16x2_bits(v0.x, v0.y), bf16x2_bits(v0.z, v0.w),
                                                    bf16x2_bits(v1.x, v1.y), bf16x2_bits(v1.z, v1.w));
  } else if constexpr (OUT == kOutF32V8) {
    st_v8(reinterpret_cast<float*>(a.out) + 8 * o, v0, v1);
  } else {
    reinterpret_cast<float4*>(a.out)[2 * o] = v0;
    reinterpret_cast<float4*>(a.out)[2 * o + 1] = v1;
  }
}

// One piece [lo, hi) of a CTA's range, as guided_piece but on octs of 8
// elements (one guidance byte, one code word, 8 output values per unit):
// two octs per lane per iteration in the nearest-rounding phase, one in
// the fine-rounding phase.
template <int FMT, int OUT, bool RZ>
__device__ __forceinline__ void guided_fq_piece(const GuidedFqArgs& a, int64_t lo, int64_t hi,
                                                const GuidedTables& tb, GuidedMode& md) {
  constexpr bool UG = kUni<FMT>;
  constexpr int OPB = kE4M3<FMT> ? 2 : 4;  // octs per block
  constexpr int OPB_LOG = kE4M3<FMT> ? 1 : 2;
  const int tid = threadIdx.x;
  const int64_t o0 = lo * OPB, o1 = hi * OPB;
  // oct counters within the piece (one CTA's share of a segment: far below
  // 2^31 octs); 32-bit ones measured faster except for NVFP4's fp32 output,
  // where they cost registers
  using Idx = std::conditional_t<kE4M3<FMT> && !kUni<FMT> && OUT != kOutBf16, int64_t, int>;
  const Idx n = (Idx)(o1 - o0);
  Idx kb = 0;
  for (; kb < n && !md.fine(); kb += 2 * kThreads) {
    uint4 xv[2];
    uint32_t sc[2], g[2];
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const Idx k = kb + u * kThreads + tid;
      const int64_t o = o0 + k;
      ok[u] = k < n && unit_ok(o, o0, o1, a.nblocks * OPB);
      if (ok[u]) {
        xv[u] = __ldg(a.x + o);
        sc[u] = __ldg(a.rec_scales + (o >> OPB_LOG));
        g[u] = __ldg(a.rec_bits + o);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t w[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
      uint32_t c = 0u, mm = 0u;
      float r = 0.0f, S = 0.0f;
      bool bad = false;
      if (ok[u]) r = fq_oct_r<FMT>(w, sc[u], g[u], tb, S, c, bad);
      if (ok[u] && r != 0.0f) c = nearest_x8<RZ, UG, true>(w[0], w[1], w[2], w[3], r, g[u], mm);
      if (md.note(mm != 0u) && mm != 0u) c = guided_x8_call<RZ, UG>(w[0], w[1], w[2], w[3], r, g[u]);
      if (ok[u]) fq_store<FMT, OUT>(a, o0 + kb + u * kThreads + tid, c, S);
      report_bad_lane(bad, a.status);
    }
  }
  for (; kb < n; kb += kThreads) {
    const Idx k = kb + tid;
    const int64_t o = o0 + k;
    const bool ok = k < n && unit_ok(o, o0, o1, a.nblocks * OPB);
    bool bad = false;
    if (ok) {
      const uint4 xv = __ldg(a.x + o);
      const uint32_t sc = __ldg(a.rec_scales + (o >> OPB_LOG)), g = __ldg(a.rec_bits + o);
      const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
      uint32_t c = 0u;
      float S = 0.0f;
      const float r = fq_oct_r<FMT>(w, sc, g, tb, S, c, bad);
      if (r != 0.0f) c = guided_x8<RZ, UG, true>(w[0], w[1], w[2], w[3], r, g);
      fq_store<FMT, OUT>(a, o, c, S);
    }
    report_bad_lane(bad, a.status);
  }
}

// OUT: kOutBf16 (one 16-B store per oct), kOutF32 (two 16-B stores),
// kOutF32V8 (one 32-B store; the host picks it only for a 32-B aligned out).
template <int FMT, class SEG, int OUT>
__global__ void __launch_bounds__(kThreads, kGuidedFqMinCtas) k_guided_fq(GuidedFqArgs a, SEG seg) {
  pdl_enter();
  constexpr bool UG = kUni<FMT>;
  __shared__ GuidedTables tb;
  int s = 0;
  int64_t lo, hi;
  if constexpr (std::is_same<SEG, SegPieces>::value) {
    seg.piece(blockIdx.x, s, lo, hi);
  } else {
    lo = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
    hi = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  }
  GuidedMode md;
  if constexpr (kE4M3<FMT>) {
    const float st = a.rec_s_t[s];
    build_tables<UG, false>(st, tb);
    build_block_tables(st, tb);
  }
  if (kE4M3<FMT> && tb.rz) guided_fq_piece<FMT, OUT, true>(a, lo, hi, tb, md);
  else guided_fq_piece<FMT, OUT, false>(a, lo, hi, tb, md);
}

// ------------------------------------------------ mismatch diagnostics
// Train/rollout mismatch statistics (TRACE summary, section
// "量子化情報キャッシュ": more than 99% of mismatches are between adjacent
// codewords).  For each element, with the rollout's recorded scale: n_r =
// nearest rounding of the train value, n_o = the rollout code, n_g = the
// guided code (recorded bit = n_o's mantissa bit); codes compare by signed
// grid index (sign ? -m3 : m3, so +0 and -0 are equal).  Accumulates
// counts[0] += #(n_r != n_o), counts[1] += #(|n_r - n_o| == 1),
// counts[2] += #(|n_r - n_o| >= 2), counts[3] += #(n_g != n_o), and the
// direction of the correction: counts[4] += #(n_r != n_o, m3(n_o) < m3(n_r))
// (toward the smaller codeword), counts[5] += #(n_r != n_o, m3(n_o) > m3(n_r)).
constexpr int kMismatchCounts = 6;

struct MismatchArgs {
  const uint4* x;
  int64_t nblocks;
  const uint8_t* rec_scales;
  const float* rec_s_t;
  const uint8_t* rec_codes;
  unsigned long long* counts;
  int32_t* status;
};

__device__ __forceinline__ int grid_index(uint32_t nib) {
  const int m = (int)(nib & 7u);
  return (nib & 8u) ? -m : m;
}

// Counts over the nibbles where code word cx differs from the rollout's co:
// with d = |index(cx) - index(co)|, cnt[0..2] += (d != 0, d == 1, d >= 2)
// and cnt[4..5] += (d != 0 and m3(co) < m3(cx), d != 0 and m3(co) > m3(cx))
// (NEAREST), or cnt[3] += (d != 0) (guided).  Equal nibbles count nothing.
template <bool NEAREST>
__device__ __forceinline__ void count_diffs(uint32_t cx, uint32_t co, uint32_t (&cnt)[kMismatchCounts]) {
  uint32_t d = cx ^ co;
  while (d) {
    const int e = (__ffs(d) - 1) >> 2;
    d &= ~(0xFu << (4 * e));
    const uint32_t nx = (cx >> (4 * e)) & 0xFu, no = (co >> (4 * e)) & 0xFu;
    const int dd = abs(grid_index(nx) - grid_index(no));
    if (NEAREST) {
      cnt[0] += dd != 0;
      cnt[1] += dd == 1;
      cnt[2] += dd >= 2;
      cnt[4] += dd != 0 && (no & 7u) < (nx & 7u);
      cnt[5] += dd != 0 && (no & 7u) > (nx & 7u);
    } else {
      cnt[3] += dd != 0;
    }
  }
}

// Per block, nearest and guided rounding of the train values on the
// recorded grid take the quantize / guided fast paths (per-segment tables
// verified against the grid's midpoints and codewords respectively; MXFP4's
// quotient is exact), falling back to exact per-element comparisons where
// no verified multiplier exists; the code words are then compared with the
// rollout's nibble-wise, and only differing nibbles are classified.
template <int FMT, class SEG>
__global__ void __launch_bounds__(kThreads, (kE4M3<FMT> && std::is_same<SEG, Seg1>::value) ? 6 : 1)
    k_mismatch(MismatchArgs a, SEG seg) {
  pdl_enter();
  constexpr bool UG = kUni<FMT>;
  constexpr int BE = kE4M3<FMT> ? 16 : 32;
  constexpr int NW = BE / 2;
  constexpr int NQ = BE / 8;
  __shared__ SegTables tmid, tcw;
  // per recorded scale byte: the multipliers of the two tables (0: exact
  // comparisons) and the block scale, one shared-memory load each per block
  __shared__ float rm_of[256], rc_of[256], s_of[256];
  const int64_t b0 = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
  const int64_t b1 = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  uint32_t cnt[kMismatchCounts] = {0u, 0u, 0u, 0u, 0u, 0u};
  int64_t lo = b0;
  bool bad = false;
  while (lo < b1) {
    const int s = seg.find(lo);
    const int64_t hi = (s + 1 < seg.count()) ? min(b1, seg.start(s + 1)) : b1;
    const float st = kE4M3<FMT> ? a.rec_s_t[s] : 0.0f;
    if constexpr (kE4M3<FMT>) {
      build_tables<UG, true, false>(st, tmid);
      build_tables<UG, false>(st, tcw);  // ends with a barrier: tmid and tcw are complete
      static_assert(kThreads == 256, "one table entry per thread");
      const uint32_t sc = threadIdx.x;
      float rm = 0.0f, rc = 0.0f;
      if ((sc >> 3) >= 1u && sc < 0x7Fu) {
        if (tmid.fast && tmid.rho[sc & 7u] != 0.0f) rm = block_rho(tmid.rho[sc & 7u], sc >> 3);
        if (tcw.fast && tcw.rho[sc & 7u] != 0.0f) rc = block_rho(tcw.rho[sc & 7u], sc >> 3);
      }
      rm_of[sc] = rm;
      rc_of[sc] = rc;
      s_of[sc] = st > 0.0f ? __fmul_rn(st, e4m3_decode(sc)) : 0.0f;
      __syncthreads();
    }
    for (int64_t blk = lo + threadIdx.x; blk < hi; blk += kThreads) {
      if (!unit_ok(blk, lo, hi, a.nblocks)) continue;
      uint32_t w[NW], cw[NQ];
#pragma unroll
      for (int q = 0; q < NW / 4; ++q) {
        const uint4 p = __ldg(a.x + (NW / 4) * blk + q);
        w[4 * q] = p.x; w[4 * q + 1] = p.y; w[4 * q + 2] = p.z; w[4 * q + 3] = p.w;
      }
      if constexpr (kE4M3<FMT>) {
        const uint2 c = __ldg(reinterpret_cast<const uint2*>(a.rec_codes) + blk);
        cw[0] = c.x; cw[1] = c.y;
      } else {
        const uint4 c = __ldg(reinterpret_cast<const uint4*>(a.rec_codes) + blk);
        cw[0] = c.x; cw[1] = c.y; cw[2] = c.z; cw[3] = c.w;
      }
      const uint32_t sc = a.rec_scales[blk];
      float S, rm = 0.0f, rc = 0.0f;
      bool rzm = false, rzc = false;
      if constexpr (kE4M3<FMT>) {
        S = s_of[sc];
        rm = rm_of[sc];
        rc = rc_of[sc];
        rzm = tmid.rz;
        rzc = tcw.rz;
      } else {
        S = __uint_as_float(sc >= 1u ? sc << 23 : 0x00400000u);
        if (sc >= 1u && sc <= 252u) rm = rc = __uint_as_float((254u - sc) << 23);  // 2^-(sc-127), exact
      }
      const uint32_t mb = block_absmax_bits(w);
      bad |= mb >= 0x7F80u;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const uint32_t* wq = &w[4 * q];
        const uint32_t co = cw[q];
        uint32_t cr = 0u, cg = 0u;
        if (rm != 0.0f) {
          cr = rzm ? cvt_words<true, UG>(wq[0], wq[1], wq[2], wq[3], rm)
                   : cvt_words<false, UG>(wq[0], wq[1], wq[2], wq[3], rm);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t h = (e & 1) ? (wq[e >> 1] >> 16) : (wq[e >> 1] & 0xFFFFu);
            const uint32_t m3 = S > 0.0f ? rtn_m3_exact<UG>(__uint_as_float((h & 0x7FFFu) << 16), S) : 0u;
            cr |= (((h >> 15) << 3) | m3) << (4 * e);
          }
        }
        // Where the train value's nearest code equals the rollout's, the
        // rollout code is one of its neighbours and carries the recorded
        // bit, so guided rounding returns it too: only octs with a differing
        // nibble can add to any count.
        if (cr == co) continue;
        if (rc != 0.0f) {
          const uint32_t gs = co & 0x11111111u;  // the rollout codes' bits, in place
          cg = rzc ? guided_x8_spread<true, UG, true>(wq[0], wq[1], wq[2], wq[3], rc, gs)
                   : guided_x8_spread<false, UG, true>(wq[0], wq[1], wq[2], wq[3], rc, gs);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t h = (e & 1) ? (wq[e >> 1] >> 16) : (wq[e >> 1] & 0xFFFFu);
            const uint32_t g = (co >> (4 * e)) & 1u;
            const uint32_t m3 = S > 0.0f ? guided_m3_exact<UG>(__uint_as_float((h & 0x7FFFu) << 16), S, g) : 0u;
            cg |= (((h >> 15) << 3) | m3) << (4 * e);
          }
        }
        count_diffs<true>(cr, co, cnt);
        count_diffs<false>(cg, co, cnt);
      }
    }
    lo = hi;
  }
  report_bad(bad, a.status);
#pragma unroll
  for (int k = 0; k < kMismatchCounts; ++k) {
    const uint32_t t = __reduce_add_sync(0xFFFFFFFFu, cnt[k]);
    if ((threadIdx.x & 31) == 0 && t) atomicAdd(a.counts + k, (unsigned long long)t);
  }
}

// ---------------------------------------------------------- dequantize
struct DequantArgs {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* s_t;
  float4* out;
  int64_t nblocks;
};

// Work unit = one quad of 4 consecutive elements (2 code bytes in, one
// 16-byte float4 out), consecutive lanes on consecutive quads, so every warp
// store covers 512 contiguous bytes.  Segment pieces are whole blocks.
template <int FMT, class SEG>
__global__ void __launch_bounds__(kThreads) k_dequant(DequantArgs a, SEG seg) {
  pdl_enter();
  constexpr int BE = kE4M3<FMT> ? 16 : 32;
  constexpr int QPB = BE / 4;  // quads per block
  constexpr int U = 4;         // quads per lane per iteration
  const int64_t b0 = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
  const int64_t b1 = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  const int tid = threadIdx.x;
  const uint16_t* codes2 = reinterpret_cast<const uint16_t*>(a.codes);
  int64_t lo = b0;
  while (lo < b1) {
    const int s = seg.find(lo);
    const int64_t hi = (s + 1 < seg.count()) ? min(b1, seg.start(s + 1)) : b1;
    const float st = kE4M3<FMT> ? a.s_t[s] : 0.0f;
    const int64_t q0 = lo * QPB, q1 = hi * QPB;
    for (int64_t qb = q0; qb < q1; qb += (int64_t)U * kThreads) {
      uint32_t cw[U], sc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t q = qb + u * kThreads + tid;
        if (q < q1 && unit_ok(q, q0, q1, a.nblocks * QPB)) {
          cw[u] = __ldg(codes2 + q);
          sc[u] = __ldg(a.scales + q / QPB);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t q = qb + u * kThreads + tid;
        if (q < q1 && unit_ok(q, q0, q1, a.nblocks * QPB)) {
          float S;
          if constexpr (kE4M3<FMT>) S = __fmul_rn(st, e4m3_decode(sc[u]));
          else S = __uint_as_float(sc[u] >= 1u ? sc[u] << 23 : 0x00400000u);
          a.out[q] = decode4_grid<kUni<FMT>>(cw[u], S);
        }
      }
    }
    lo = hi;
  }
}

// Dequantize with 8 elements per lane (one code word in, one 32-byte store
// out, so every warp store covers 1 KiB contiguous); the host picks it when
// out is 32-B aligned.
template <int FMT, class SEG>
__global__ void __launch_bounds__(kThreads) k_dequant8(DequantArgs a, SEG seg) {
  pdl_enter();
  constexpr int BE = kE4M3<FMT> ? 16 : 32;
  constexpr int OPB = BE / 8;  // octs per block
  constexpr int U = 4;         // octs per lane per iteration
  const int64_t b0 = cta_begin(blockIdx.x, gridDim.x, a.nblocks);
  const int64_t b1 = cta_begin(blockIdx.x + 1, gridDim.x, a.nblocks);
  const int tid = threadIdx.x;
  const uint32_t* codes4 = reinterpret_cast<const uint32_t*>(a.codes);
  float* out = reinterpret_cast<float*>(a.out);
  int64_t lo = b0;
  while (lo < b1) {
    const int s = seg.find(lo);
    const int64_t hi = (s + 1 < seg.count()) ? min(b1, seg.start(s + 1)) : b1;
    const float st = kE4M3<FMT> ? a.s_t[s] : 0.0f;
    const int64_t o0 = lo * OPB, o1 = hi * OPB;
    for (int64_t ob = o0; ob < o1; ob += (int64_t)U * kThreads) {
      uint32_t cw[U], sc[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t o = ob + u * kThreads + tid;
        if (o < o1 && unit_ok(o, o0, o1, a.nblocks * OPB)) {
          cw[u] = __ldg(codes4 + o);
          sc[u] = __ldg(a.scales + o / OPB);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t o = ob + u * kThreads + tid;
        if (o < o1 && unit_ok(o, o0, o1, a.nblocks * OPB)) {
          float S;
          if constexpr (kE4M3<FMT>) S = __fmul_rn(st, e4m3_decode(sc[u]));
          else S = __uint_as_float(sc[u] >= 1u ? sc[u] << 23 : 0x00400000u);
          float4 v0, v1;
          decode8_grid<kUni<FMT>>(cw[u], S, v0, v1);
          st_v8(out + 8 * o, v0, v1);
        }
      }
    }
    lo = hi;
  }
}

// ------------------------------------------------------- pack / unpack
// Units of 32 elements: 16 code bytes -> 4 guidance bytes.  A trailing half
// unit (16 elements, when rows*cols % 32 == 16) is done by the last thread.
__global__ void __launch_bounds__(kThreads) k_pack(const uint8_t* __restrict__ codes, uint8_t* bits,
                                                   int64_t nunits, int tail) {
  pdl_enter();
  constexpr int U = 4;
  const int64_t u0 = cta_begin(blockIdx.x, gridDim.x, nunits);
  const int64_t u1 = cta_begin(blockIdx.x + 1, gridDim.x, nunits);
  const uint4* c4 = reinterpret_cast<const uint4*>(codes);
  for (int64_t ub = u0; ub < u1; ub += (int64_t)U * kThreads) {
    uint4 c[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t u = ub + k * kThreads + threadIdx.x;
      if (u < u1 && unit_ok(u, u0, u1, nunits)) c[k] = __ldg(c4 + u);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t u = ub + k * kThreads + threadIdx.x;
      if (u < u1 && unit_ok(u, u0, u1, nunits))
        reinterpret_cast<uint32_t*>(bits)[u] = nibble_lsbs(c[k].x) | (nibble_lsbs(c[k].y) << 8) |
                                               (nibble_lsbs(c[k].z) << 16) | (nibble_lsbs(c[k].w) << 24);
    }
  }
  if (tail && blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + 16 * nunits);
    reinterpret_cast<uint16_t*>(bits)[2 * nunits] = (uint16_t)(nibble_lsbs(c.x) | (nibble_lsbs(c.y) << 8));
  }
}

// bits of one byte -> 8 bytes of 0/1 (bit k -> byte k)
__device__ __forceinline__ uint2 spread8(uint32_t b) {
  uint32_t o[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t nib = (b >> (4 * q)) & 0xFu;
    o[q] = (nib & 1u) | ((nib & 2u) << 7) | ((nib & 4u) << 14) | ((nib & 8u) << 21);
  }
  return make_uint2(o[0], o[1]);
}

// Units of 16 elements: 2 guidance bytes -> 16 bytes of 0/1; consecutive
// lanes on consecutive units, so every warp store covers 512 contiguous bytes.
__global__ void __launch_bounds__(kThreads) k_unpack(const uint8_t* __restrict__ bits, uint8_t* mant,
                                                     int64_t nunits) {
  pdl_enter();
  constexpr int U = 4;
  const int64_t u0 = cta_begin(blockIdx.x, gridDim.x, nunits);
  const int64_t u1 = cta_begin(blockIdx.x + 1, gridDim.x, nunits);
  const uint16_t* b2 = reinterpret_cast<const uint16_t*>(bits);
  uint4* out = reinterpret_cast<uint4*>(mant);
  for (int64_t ub = u0; ub < u1; ub += (int64_t)U * kThreads) {
    uint32_t b[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t u = ub + k * kThreads + threadIdx.x;
      if (u < u1 && unit_ok(u, u0, u1, nunits)) b[k] = __ldg(b2 + u);
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t u = ub + k * kThreads + threadIdx.x;
      if (u < u1 && unit_ok(u, u0, u1, nunits)) {
        const uint2 lo = spread8(b[k] & 0xFFu), hi = spread8(b[k] >> 8);
        out[u] = make_uint4(lo.x, lo.y, hi.x, hi.y);
      }
    }
  }
}

// ------------------------------------------------- tiled scale layout
// Block scales rearranged for block-scaled FP4 GEMMs (the cuBLAS
// documentation's "1D Block Scaling Factors Layout"): the [rows, nb] scale
// matrix, zero-padded to 128-row x 4-column tiles, tiles in row-major
// order, 512 bytes each, entry (r, c) of a tile at byte (r % 32) * 16 +
// (r / 32) * 4 + c.  One lane writes one 16-byte line of a tile: row
// i = r % 32 of its four 32-row groups, 4 columns each.
__global__ void __launch_bounds__(kThreads) k_swizzle(const uint8_t* __restrict__ scales, int64_t rows, int64_t nb,
                                                      int64_t ntc, int64_t nlines, uint4* out) {
  pdl_enter();
  for (int64_t l = (int64_t)blockIdx.x * kThreads + threadIdx.x; l < nlines; l += (int64_t)gridDim.x * kThreads) {
    const int64_t tile = l >> 5;
    const int64_t i = l & 31;
    const int64_t r0 = (tile / ntc) * 128 + i, c0 = (tile % ntc) * 4;
    uint32_t word[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t r = r0 + 32 * j;
      uint32_t v = 0u;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (r < rows && c0 + c < nb && unit_ok(r * nb + c0 + c, 0, rows * nb, rows * nb))
          v |= (uint32_t)__ldg(scales + r * nb + c0 + c) << (8 * c);
      word[j] = v;
    }
    if (unit_ok(l, 0, nlines, nlines)) out[l] = make_uint4(word[0], word[1], word[2], word[3]);
  }
}

}  // namespace tf4
