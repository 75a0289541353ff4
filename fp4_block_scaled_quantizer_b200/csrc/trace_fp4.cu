// trace_fp4.cu -- C ABI of the trace_fp4 library (see include/trace_fp4.h):
// argument validation, launch geometry, and the kernel launches.
#include <cuda_runtime.h>

#include <climits>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/trace_fp4.h"
#include "tf4_kernels.cuh"

namespace {

using tf4::kThreads;

struct Shape {
  int fmt;
  int be;         // elements per quantization block
  int64_t rows, cols, n, nblocks;
  int nseg;
  const int64_t* off;
};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Formats with an fp32 tensor scale (and hence segments and a workspace).
bool has_tensor_scale(int fmt) { return fmt != TF4_MXFP4; }

// Calls f with the format as a compile-time constant.
template <class F>
void by_format(int fmt, F&& f) {
  if (fmt == TF4_NVFP4) f(std::integral_constant<int, TF4_NVFP4>{});
  else if (fmt == TF4_UFP4) f(std::integral_constant<int, TF4_UFP4>{});
  else f(std::integral_constant<int, TF4_MXFP4>{});
}

tf4_status check_desc(const tf4_desc* d, Shape* sh) {
  if (!d) return TF4_ERR_INVALID_ARG;
  if (d->fmt != TF4_NVFP4 && d->fmt != TF4_MXFP4 && d->fmt != TF4_UFP4) return TF4_ERR_INVALID_ARG;
  const int be = d->fmt == TF4_MXFP4 ? 32 : 16;
  if (d->rows < 0 || d->cols <= 0 || d->cols % be != 0) return TF4_ERR_SHAPE;
  if (d->rows > 0 && d->cols > (int64_t)(LLONG_MAX / 64) / d->rows) return TF4_ERR_SHAPE;
  const int nseg = d->num_segments;
  if (nseg < 1 || nseg > TF4_MAX_SEGMENTS) return TF4_ERR_INVALID_ARG;
  if (d->fmt == TF4_MXFP4 && nseg != 1) return TF4_ERR_INVALID_ARG;
  if (nseg > 1 && !d->seg_row_offsets) return TF4_ERR_INVALID_ARG;
  if (d->seg_row_offsets) {
    const int64_t* o = d->seg_row_offsets;
    if (o[0] != 0 || o[nseg] != d->rows) return TF4_ERR_INVALID_ARG;
    for (int s = 0; s < nseg; ++s)
      if (o[s + 1] < o[s]) return TF4_ERR_INVALID_ARG;
    if (nseg > 1 && d->rows > INT_MAX) return TF4_ERR_SHAPE;
  }
  sh->fmt = d->fmt;
  sh->be = be;
  sh->rows = d->rows;
  sh->cols = d->cols;
  sh->n = d->rows * d->cols;
  sh->nblocks = sh->n / be;
  sh->nseg = nseg;
  sh->off = d->seg_row_offsets;
  return TF4_OK;
}

tf4::SegN make_segn(const Shape& sh) {
  tf4::SegN s;
  std::memset(&s, 0, sizeof s);
  s.nseg = sh.nseg;
  s.bpr = sh.cols / sh.be;
  for (int k = 0; k <= sh.nseg; ++k) s.off[k] = (int32_t)sh.off[k];
  return s;
}

// Ragged segments for the guided kernels: each non-empty segment gets its
// own CTAs, about grid_target x its share of the blocks (at least one, at
// most one per block).
tf4::SegPieces make_segpieces(const Shape& sh, int64_t grid_target) {
  tf4::SegPieces p;
  std::memset(&p, 0, sizeof p);
  p.nseg = sh.nseg;
  p.bpr = sh.cols / sh.be;
  for (int k = 0; k <= sh.nseg; ++k) p.off[k] = (int32_t)sh.off[k];
  const int64_t n = sh.nblocks > 0 ? sh.nblocks : 1;
  int64_t c = 0;
  for (int k = 0; k < sh.nseg; ++k) {
    p.cta[k] = (int32_t)c;
    const int64_t len = (int64_t)(sh.off[k + 1] - sh.off[k]) * p.bpr;
    if (len > 0) {
      int64_t cnt = (len * grid_target + n / 2) / n;
      cnt = cnt < 1 ? 1 : (cnt > len ? len : cnt);
      c += cnt;
    }
  }
  p.cta[sh.nseg] = (int32_t)c;
  return p;
}

bool multi(const Shape& sh) { return sh.nseg > 1; }

int sm_count() {
  static int cache[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Resident CTAs per SM of `kernel` on the current device (cached).
int occupancy(const void* kernel) {
  struct Entry { int dev; const void* k; int occ; };
  static Entry cache[256];
  static int used = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].dev == dev && cache[i].k == kernel) return cache[i].occ;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, 0) != cudaSuccess || occ <= 0) {
    cudaGetLastError();
    occ = 1;
  }
  if (used < 256) cache[used++] = Entry{dev, kernel, occ};
  return occ;
}

// Grid = waves x SMs x resident CTAs of `kernel`: up to 4 waves while every
// CTA still gets at least 32768 elements (2048 units of unit_elems = 16;
// MXFP4 blocks count 32 each, which gives MXFP4 the same number of waves as
// NVFP4 on one tensor -- 1 -> 3 waves on a 256 MiB tensor made its
// dequantize and fused fake-quant 9-14% faster); smaller ranges let CTAs
// that finish early pick up the next wave's ranges, which shortens the tail
// of a single wave of equal ranges; never more CTAs than units.
template <class K>
int64_t wave_grid(K kernel, int64_t units, int unit_elems = 16) {
  const int64_t wave = (int64_t)sm_count() * occupancy(reinterpret_cast<const void*>(kernel));
  int64_t waves = units * unit_elems / (wave * 2048 * 16);
  waves = waves < 1 ? 1 : (waves > 4 ? 4 : waves);
  const int64_t g = wave * waves;
  return units < g ? (units > 0 ? units : 1) : g;
}

tf4_status launched() {
  return cudaGetLastError() == cudaSuccess ? TF4_OK : TF4_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may be
// scheduled while the previous grid in the stream is finishing; every
// kernel of the library waits for that grid (griddepcontrol.wait) before
// touching memory, so ordering is as for a plain launch, minus the launch
// gap.  Errors are left for launched().
template <typename... KArgs, typename... Args>
void launch_k(void (*kernel)(KArgs...), int64_t grid, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

size_t ws_bytes_for(const Shape& sh) {
  if (!has_tensor_scale(sh.fmt)) return 0;
  return ((size_t)(sh.nseg + 1) * sizeof(uint32_t) + 255) & ~(size_t)255;
}

// Quantize grid of the tensor-scale formats: shared by the amax pass and
// the quantize pass so that both cover the same byte range per CTA.
template <int FMT, int MODE>
int64_t nvfp4_grid(const Shape& sh) {
  return multi(sh) ? wave_grid(tf4::k_quant<FMT, MODE, tf4::SegN>, sh.nblocks)
                   : wave_grid(tf4::k_quant<FMT, MODE, tf4::Seg1>, sh.nblocks);
}

// The amax pass; s_t_out (if not NULL) receives the tensor scale of FMT's grid.
template <int FMT>
tf4_status launch_amax(const Shape& sh, int64_t grid, const void* x, uint32_t* ws, float* s_t_out,
                       float* amax_out, int32_t* status, cudaStream_t st) {
  constexpr bool U = tf4::kUni<FMT>;
  const uint4* x4 = static_cast<const uint4*>(x);
  // the amax pass works on 16-element blocks whatever the format
  const int64_t nb16 = sh.n / 16;
  if (multi(sh)) {
    tf4::SegN seg = make_segn(sh);
    seg.bpr = sh.cols / 16;
    launch_k(tf4::k_amax<tf4::SegN, U>, grid, st, x4, nb16, seg, ws, s_t_out, amax_out, status);
  } else {
    launch_k(tf4::k_amax<tf4::Seg1, U>, grid, st, x4, nb16, tf4::Seg1{}, ws, s_t_out, amax_out, status);
  }
  return launched();
}

// Tensors of at most this many elements (64 MiB of bf16, half the L2)
// with one segment are captured by the single-launch kernel; larger ones
// by the amax launch and the quantize launch.
constexpr int64_t kFusedMaxElems = int64_t(1) << 25;
// Bound of the single-launch kernel's grid-wide wait (ns of %globaltimer):
// its amax phase over 64 MiB takes about 10 us.
constexpr uint64_t kFusedWaitNs = 100000000ull;

// Resident CTAs per SM of `kernel` with `smem` bytes of dynamic shared
// memory on the current device (not cached).
int occupancy_smem(const void* kernel, size_t smem) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, smem) != cudaSuccess || occ <= 0) {
    cudaGetLastError();
    occ = 0;
  }
  return occ;
}

// Dynamic shared memory the staged single-launch capture may use per CTA
// (the default limit, no opt-in needed).
constexpr size_t kStageMaxBytes = 48 * 1024;

// The single-launch capture (k_quant_fused): a cooperative launch, so that
// every CTA is resident while the CTAs wait for one another; at least 256
// quantization blocks per CTA.  When every CTA's range of x fits in
// kStageMaxBytes of shared memory at full residency, the staged variant
// keeps it there between the two phases.
template <int FMT, int MODE>
tf4_status launch_fused(const Shape& sh, const tf4::QuantArgs& a, uint32_t* ws, const tf4::PhiloxKeys& pk,
                        cudaStream_t st) {
  auto plain = tf4::k_quant_fused<FMT, MODE, false>;
  auto staged = tf4::k_quant_fused<FMT, MODE, true>;
  const int64_t resident = (int64_t)sm_count() * occupancy(reinterpret_cast<const void*>(plain));
  int64_t g = (sh.nblocks + 255) / 256;
  g = g < resident ? g : resident;
  g = g < 1 ? 1 : g;
  const size_t stage_bytes = (size_t)((sh.nblocks + g - 1) / g) * 32;  // 16 bf16 per block
  bool use_stage = stage_bytes <= kStageMaxBytes;
  if (use_stage) {
    const int64_t r2 = (int64_t)sm_count() * occupancy_smem(reinterpret_cast<const void*>(staged), stage_bytes);
    use_stage = r2 >= g;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)g);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = use_stage ? stage_bytes : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (use_stage) cudaLaunchKernelEx(&cfg, staged, a, ws, pk, kFusedWaitNs);
  else cudaLaunchKernelEx(&cfg, plain, a, ws, pk, kFusedWaitNs);
  return launched();
}

template <int MODE>
tf4_status quantize_impl(const tf4_desc* d, const void* x, uint64_t seed, const float* amax_in,
                         uint8_t* codes, uint8_t* scales, float* s_t, uint8_t* bits, void* ws,
                         size_t ws_bytes, int32_t* status, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(d, &sh);
  if (e != TF4_OK) return e;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool nv = has_tensor_scale(sh.fmt);
  if (nv && !s_t) return TF4_ERR_INVALID_ARG;
  if (nv && (!aligned(s_t, 4) || (amax_in && !aligned(amax_in, 4)))) return TF4_ERR_ALIGN;
  if (status && !aligned(status, 4)) return TF4_ERR_ALIGN;
  if (sh.n == 0) {
    if (nv) return cudaMemsetAsync(s_t, 0, sizeof(float) * sh.nseg, st) == cudaSuccess ? TF4_OK : TF4_ERR_CUDA;
    return TF4_OK;
  }
  if (!x || !codes || !scales) return TF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || (bits && !aligned(bits, 4))) return TF4_ERR_ALIGN;
  if (nv && !amax_in) {
    if (!ws) return TF4_ERR_WORKSPACE;
    if (!aligned(ws, 4)) return TF4_ERR_ALIGN;
    if (ws_bytes < ws_bytes_for(sh)) return TF4_ERR_WORKSPACE;
  }
  tf4::QuantArgs a;
  a.x = static_cast<const uint4*>(x);
  a.nblocks = sh.nblocks;
  a.codes = codes;
  a.scales = scales;
  a.bits = bits;
  a.seed = seed;
  tf4::PhiloxKeys pk;
  tf4::philox_schedule(seed, pk.ks);
  a.status = status;
  a.s_t_out = s_t;
  if (nv) {
    by_format(sh.fmt, [&](auto f) {
      constexpr int FMT = decltype(f)::value;
      if constexpr (tf4::kE4M3<FMT>) {
        const int64_t grid = nvfp4_grid<FMT, MODE>(sh);
        if constexpr (MODE != tf4::kSR) {
          if (!amax_in && !multi(sh) && sh.n <= kFusedMaxElems) {
            e = launch_fused<FMT, MODE>(sh, a, static_cast<uint32_t*>(ws), pk, st);
            return;
          }
        }
        if (amax_in) {
          a.st_src = amax_in;
          a.st_from_amax = 1;
        } else {
          e = launch_amax<FMT>(sh, grid, x, static_cast<uint32_t*>(ws), s_t, nullptr, status, st);
          if (e != TF4_OK) return;
          a.st_src = s_t;
          a.st_from_amax = 0;
        }
        if (multi(sh))
          launch_k(tf4::k_quant<FMT, MODE, tf4::SegN>, grid, st, a, make_segn(sh), pk);
        else
          launch_k(tf4::k_quant<FMT, MODE, tf4::Seg1>, grid, st, a, tf4::Seg1{}, pk);
      }
    });
    if (e != TF4_OK) return e;
  } else {
    a.st_src = nullptr;
    a.st_from_amax = 0;
    a.s_t_out = nullptr;
    const int64_t grid = wave_grid(tf4::k_quant<TF4_MXFP4, MODE, tf4::Seg1>, sh.nblocks, sh.be);
    launch_k(tf4::k_quant<TF4_MXFP4, MODE, tf4::Seg1>, grid, st, a, tf4::Seg1{}, pk);
  }
  return launched();
}

// Scratch of the allocation-free capture: the amax pass's per-segment
// maxima and its completion counter, in a fixed device array owned by the
// library (zero at load; cleared again by every call that uses it).  Sized
// like a workspace for TF4_NOALLOC_MAX_SEGMENTS segments (whole 256-byte
// units: 1280 bytes).
constexpr int kNoAllocWords = ((TF4_NOALLOC_MAX_SEGMENTS + 1) * 4 + 255) / 256 * 64;
static __device__ __align__(256) uint32_t tf4_noalloc_scratch[kNoAllocWords];

// Device address of tf4_noalloc_scratch on device `dev`, which must be the
// current device: looked up once per device (with that device current) and
// cached.
uint32_t* noalloc_scratch(int dev) {
  static uint32_t* addr[128] = {nullptr};
  static std::mutex mu;
  if (dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, tf4_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<uint32_t*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" {

size_t tf4_workspace_bytes(const tf4_desc* desc) {
  Shape sh;
  if (check_desc(desc, &sh) != TF4_OK) return 0;
  return ws_bytes_for(sh);
}

size_t tf4_codes_bytes(const tf4_desc* desc) {
  Shape sh;
  return check_desc(desc, &sh) == TF4_OK ? (size_t)(sh.n / 2) : 0;
}

size_t tf4_scales_bytes(const tf4_desc* desc) {
  Shape sh;
  return check_desc(desc, &sh) == TF4_OK ? (size_t)sh.nblocks : 0;
}

size_t tf4_guidance_bytes(const tf4_desc* desc) {
  Shape sh;
  return check_desc(desc, &sh) == TF4_OK ? (size_t)(sh.n / 8) : 0;
}

size_t tf4_record_bytes(const tf4_desc* desc, int with_codes) {
  Shape sh;
  if (check_desc(desc, &sh) != TF4_OK) return 0;
  size_t b = with_codes ? (size_t)(sh.n / 2) : (size_t)(sh.n / 8);
  b += (size_t)sh.nblocks;
  if (has_tensor_scale(sh.fmt)) b += sizeof(float) * (size_t)sh.nseg;
  return b;
}

tf4_status tf4_segment_amax(const tf4_desc* desc, const void* x, float* amax, void* ws, size_t ws_bytes,
                            int32_t* status, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (!has_tensor_scale(sh.fmt)) return TF4_ERR_INVALID_ARG;
  if (!amax) return TF4_ERR_INVALID_ARG;
  if (!aligned(amax, 4) || (status && !aligned(status, 4))) return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (sh.n == 0)
    return cudaMemsetAsync(amax, 0, sizeof(float) * sh.nseg, st) == cudaSuccess ? TF4_OK : TF4_ERR_CUDA;
  if (!x) return TF4_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return TF4_ERR_ALIGN;
  if (!ws) return TF4_ERR_WORKSPACE;
  if (!aligned(ws, 4)) return TF4_ERR_ALIGN;
  if (ws_bytes < ws_bytes_for(sh)) return TF4_ERR_WORKSPACE;
  // the maxima do not depend on the grid; size the grid like NVFP4's quantize pass
  return launch_amax<TF4_NVFP4>(sh, nvfp4_grid<TF4_NVFP4, tf4::kRTN>(sh), x, static_cast<uint32_t*>(ws), nullptr,
                                amax, status, st);
}

tf4_status tf4_quantize_rtn(const tf4_desc* desc, const void* x, const float* amax_in, uint8_t* codes,
                            uint8_t* scales, float* s_t, void* ws, size_t ws_bytes, int32_t* status,
                            tf4_stream_t stream) {
  return quantize_impl<tf4::kRTN>(desc, x, 0, amax_in, codes, scales, s_t, nullptr, ws, ws_bytes, status,
                                  stream);
}

tf4_status tf4_quantize_sr(const tf4_desc* desc, const void* x, uint64_t seed, const float* amax_in,
                           uint8_t* codes, uint8_t* scales, float* s_t, void* ws, size_t ws_bytes,
                           int32_t* status, tf4_stream_t stream) {
  return quantize_impl<tf4::kSR>(desc, x, seed, amax_in, codes, scales, s_t, nullptr, ws, ws_bytes, status,
                                 stream);
}

tf4_status tf4_quantize_capture(const tf4_desc* desc, const void* x, const float* amax_in, uint8_t* codes,
                                uint8_t* scales, float* s_t, uint8_t* bits, void* ws, size_t ws_bytes,
                                int32_t* status, tf4_stream_t stream) {
  if (!bits)
    return quantize_impl<tf4::kRTN>(desc, x, 0, amax_in, codes, scales, s_t, nullptr, ws, ws_bytes, status,
                                    stream);
  return quantize_impl<tf4::kCAPTURE>(desc, x, 0, amax_in, codes, scales, s_t, bits, ws, ws_bytes, status,
                                      stream);
}

// Layers of at least this many elements (256 MiB of bf16) are captured by
// one launch pair per layer; smaller layers by one pair for the whole batch
// (measured on B200: batching wins up to 128 MiB layers -- by 1.35x there
// and by 3-9x for 4-16 MiB layers -- and loses about 5% at 512 MiB).
constexpr int64_t kBatchPerLayerElems = int64_t(1) << 27;

size_t tf4_workspace_bytes_batched(int32_t num_layers) {
  if (num_layers < 1 || num_layers > TF4_MAX_BATCH) return 0;
  return ((size_t)(num_layers + 1) * sizeof(uint32_t) + 255) & ~(size_t)255;
}

tf4_status tf4_quantize_capture_batched(const tf4_desc* desc, int32_t nl, const void* const* x, uint8_t* codes,
                                        uint8_t* scales, float* s_t, int32_t keep, uint8_t* info_bits, void* ws,
                                        size_t ws_bytes, int32_t* status, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.nseg != 1) return TF4_ERR_INVALID_ARG;
  if (nl < 1 || nl > TF4_MAX_BATCH || !x) return TF4_ERR_INVALID_ARG;
  if (keep < 0 || keep > nl || ((keep > 0) != (info_bits != nullptr))) return TF4_ERR_INVALID_ARG;
  const bool nv = has_tensor_scale(sh.fmt);
  if (nv && !s_t) return TF4_ERR_INVALID_ARG;
  if ((nv && !aligned(s_t, 4)) || (status && !aligned(status, 4))) return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (sh.n == 0) {
    if (nv) return cudaMemsetAsync(s_t, 0, sizeof(float) * nl, st) == cudaSuccess ? TF4_OK : TF4_ERR_CUDA;
    return TF4_OK;
  }
  if (!codes || !scales) return TF4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || (info_bits && !aligned(info_bits, 4))) return TF4_ERR_ALIGN;
  for (int k = 0; k < nl; ++k) {
    if (!x[k]) return TF4_ERR_INVALID_ARG;
    if (!aligned(x[k], 16)) return TF4_ERR_ALIGN;
  }
  if (nv) {
    if (!ws) return TF4_ERR_WORKSPACE;
    if (!aligned(ws, 4)) return TF4_ERR_ALIGN;
    if (ws_bytes < tf4_workspace_bytes_batched(nl)) return TF4_ERR_WORKSPACE;
  }
  if (sh.n >= kBatchPerLayerElems) {
    // Large layers: the per-layer launch pair is as fast as it gets (the
    // quantize pass re-reads the amax pass's last blocks from L2, and the
    // single-tensor kernels run at higher occupancy); launch gaps are
    // negligible next to a layer's run time.
    const int64_t first_kept = nl - keep;
    for (int k = 0; k < nl; ++k) {
      uint8_t* bk = k >= first_kept ? info_bits + (size_t)(k - first_kept) * (size_t)(sh.n / 8) : nullptr;
      e = tf4_quantize_capture(desc, x[k], nullptr, codes + (size_t)k * (size_t)(sh.n / 2),
                               scales + (size_t)k * (size_t)sh.nblocks, nv ? s_t + k : nullptr, bk, ws, ws_bytes,
                               status, stream);
      if (e != TF4_OK) return e;
    }
    return TF4_OK;
  }
  tf4::SegBatch sb;
  std::memset(&sb, 0, sizeof sb);
  sb.nlayers = nl;
  sb.first_kept = nl - keep;
  sb.bpl = sh.nblocks;
  sb.units_per_block = sh.be / 8;
  sb.bits_per_block = sh.be / 8;
  for (int k = 0; k < nl; ++k) sb.x[k] = static_cast<const uint4*>(x[k]);
  const int64_t total = sh.nblocks * nl;
  tf4::QuantArgs a;
  a.x = nullptr;
  a.nblocks = total;
  a.codes = codes;
  a.scales = scales;
  a.bits = info_bits;
  a.seed = 0;
  tf4::PhiloxKeys pk;
  tf4::philox_schedule(0, pk.ks);
  a.status = status;
  a.s_t_out = s_t;
  a.st_src = s_t;
  a.st_from_amax = 0;
  if (nv) {
    by_format(sh.fmt, [&](auto f) {
      constexpr int FMT = decltype(f)::value;
      if constexpr (tf4::kE4M3<FMT>) {
        const int64_t grid = wave_grid(tf4::k_quant<FMT, tf4::kCAPTURE, tf4::SegBatch>, total);
        launch_k(tf4::k_amax<tf4::SegBatch, tf4::kUni<FMT>>, grid, st, nullptr, total, sb,
                 static_cast<uint32_t*>(ws), s_t, nullptr, status);
        if ((e = launched()) != TF4_OK) return;
        launch_k(tf4::k_quant<FMT, tf4::kCAPTURE, tf4::SegBatch>, grid, st, a, sb, pk);
      }
    });
    if (e != TF4_OK) return e;
  } else {
    a.s_t_out = nullptr;
    a.st_src = nullptr;
    const int64_t grid = wave_grid(tf4::k_quant<TF4_MXFP4, tf4::kCAPTURE, tf4::SegBatch>, total, 32);
    launch_k(tf4::k_quant<TF4_MXFP4, tf4::kCAPTURE, tf4::SegBatch>, grid, st, a, sb, pk);
  }
  return launched();
}

tf4_status tf4_quantize_guided(const tf4_desc* desc, const void* x, const uint8_t* rec_scales,
                               const float* rec_s_t, const uint8_t* rec_bits, uint8_t* codes, int32_t* status,
                               tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  const bool nv = has_tensor_scale(sh.fmt);
  if (!x || !rec_scales || !rec_bits || !codes || (nv && !rec_s_t)) return TF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(rec_bits, 4) || (nv && !aligned(rec_s_t, 4)) ||
      (status && !aligned(status, 4)))
    return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tf4::GuidedArgs a;
  a.x = static_cast<const uint4*>(x);
  a.nblocks = sh.nblocks;
  a.rec_scales = rec_scales;
  a.rec_s_t = rec_s_t;
  a.rec_bits = rec_bits;
  a.codes = codes;
  a.status = status;
  by_format(sh.fmt, [&](auto f) {
    constexpr int FMT = decltype(f)::value;
    if constexpr (tf4::kE4M3<FMT>) {
      if (multi(sh)) {
        const tf4::SegPieces p =
            make_segpieces(sh, wave_grid(tf4::k_guided<FMT, tf4::SegPieces>, sh.nblocks, sh.be));
        launch_k(tf4::k_guided<FMT, tf4::SegPieces>, p.cta[p.nseg], st, a, p);
        return;
      }
    }
    const int64_t g = wave_grid(tf4::k_guided<FMT, tf4::Seg1>, sh.nblocks, sh.be);
    launch_k(tf4::k_guided<FMT, tf4::Seg1>, g, st, a, tf4::Seg1{});
  });
  return launched();
}

tf4_status tf4_guided_fake_quant(const tf4_desc* desc, const void* x, const uint8_t* rec_scales,
                                 const float* rec_s_t, const uint8_t* rec_bits, uint8_t* codes, void* out,
                                 int out_bf16, int32_t* status, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  const bool nv = has_tensor_scale(sh.fmt);
  if (!x || !rec_scales || !rec_bits || !out || (nv && !rec_s_t)) return TF4_ERR_INVALID_ARG;
  if (out_bf16 != 0 && out_bf16 != 1) return TF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16) || !aligned(rec_bits, 4) || (codes && !aligned(codes, 16)) ||
      (nv && !aligned(rec_s_t, 4)) || (status && !aligned(status, 4)))
    return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tf4::GuidedFqArgs a;
  a.x = static_cast<const uint4*>(x);
  a.nblocks = sh.nblocks;
  a.rec_scales = rec_scales;
  a.rec_s_t = rec_s_t;
  a.rec_bits = rec_bits;
  a.codes = codes;
  a.out = out;
  a.status = status;
#define TF4_LAUNCH_FQ(FMT, SEG, OUT, segv)                                            \
  do {                                                                                \
    const int64_t g = wave_grid(tf4::k_guided_fq<FMT, SEG, OUT>, sh.nblocks, sh.be);   \
    launch_k(tf4::k_guided_fq<FMT, SEG, OUT>, g, st, a, segv);                        \
  } while (0)
#define TF4_LAUNCH_FQ_PIECES(FMT, OUT)                                                \
  do {                                                                                \
    const tf4::SegPieces p = make_segpieces(                                          \
        sh, wave_grid(tf4::k_guided_fq<FMT, tf4::SegPieces, OUT>, sh.nblocks, sh.be)); \
    launch_k(tf4::k_guided_fq<FMT, tf4::SegPieces, OUT>, p.cta[p.nseg], st, a, p);     \
  } while (0)
  // fp32 output: one 32-byte store per 8 elements when out allows it
  const int mode = out_bf16 ? tf4::kOutBf16 : (aligned(out, 32) ? tf4::kOutF32V8 : tf4::kOutF32);
  by_format(sh.fmt, [&](auto f) {
    constexpr int FMT = decltype(f)::value;
    if constexpr (tf4::kE4M3<FMT>) {
      if (multi(sh)) {
        if (mode == tf4::kOutBf16) TF4_LAUNCH_FQ_PIECES(FMT, tf4::kOutBf16);
        else if (mode == tf4::kOutF32V8) TF4_LAUNCH_FQ_PIECES(FMT, tf4::kOutF32V8);
        else TF4_LAUNCH_FQ_PIECES(FMT, tf4::kOutF32);
        return;
      }
    }
    if (mode == tf4::kOutBf16) TF4_LAUNCH_FQ(FMT, tf4::Seg1, tf4::kOutBf16, tf4::Seg1{});
    else if (mode == tf4::kOutF32V8) TF4_LAUNCH_FQ(FMT, tf4::Seg1, tf4::kOutF32V8, tf4::Seg1{});
    else TF4_LAUNCH_FQ(FMT, tf4::Seg1, tf4::kOutF32, tf4::Seg1{});
  });
#undef TF4_LAUNCH_FQ
#undef TF4_LAUNCH_FQ_PIECES
  return launched();
}

tf4_status tf4_mismatch_stats(const tf4_desc* desc, const void* x, const uint8_t* rec_scales, const float* rec_s_t,
                              const uint8_t* rec_codes, unsigned long long* counts, int32_t* status,
                              tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (!counts) return TF4_ERR_INVALID_ARG;
  if (!aligned(counts, 8) || (status && !aligned(status, 4))) return TF4_ERR_ALIGN;
  if (sh.n == 0) return TF4_OK;
  const bool nv = has_tensor_scale(sh.fmt);
  if (!x || !rec_scales || !rec_codes || (nv && !rec_s_t)) return TF4_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(rec_codes, 16) || (nv && !aligned(rec_s_t, 4))) return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tf4::MismatchArgs a;
  a.x = static_cast<const uint4*>(x);
  a.nblocks = sh.nblocks;
  a.rec_scales = rec_scales;
  a.rec_s_t = rec_s_t;
  a.rec_codes = rec_codes;
  a.counts = counts;
  a.status = status;
  by_format(sh.fmt, [&](auto f) {
    constexpr int FMT = decltype(f)::value;
    if constexpr (tf4::kE4M3<FMT>) {
      if (multi(sh)) {
        const int64_t g = wave_grid(tf4::k_mismatch<FMT, tf4::SegN>, sh.nblocks, sh.be);
        launch_k(tf4::k_mismatch<FMT, tf4::SegN>, g, st, a, make_segn(sh));
        return;
      }
    }
    const int64_t g = wave_grid(tf4::k_mismatch<FMT, tf4::Seg1>, sh.nblocks, sh.be);
    launch_k(tf4::k_mismatch<FMT, tf4::Seg1>, g, st, a, tf4::Seg1{});
  });
  return launched();
}

tf4_status tf4_dequantize(const tf4_desc* desc, const uint8_t* codes, const uint8_t* scales, const float* s_t,
                          float* out, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  const bool nv = has_tensor_scale(sh.fmt);
  if (!codes || !scales || !out || (nv && !s_t)) return TF4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(out, 16) || (nv && !aligned(s_t, 4))) return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  tf4::DequantArgs a;
  a.codes = codes;
  a.scales = scales;
  a.s_t = s_t;
  a.out = reinterpret_cast<float4*>(out);
  a.nblocks = sh.nblocks;
  // 8 elements and one 32-byte store per lane when out allows it
  const bool v8 = aligned(out, 32);
  by_format(sh.fmt, [&](auto f) {
    constexpr int FMT = decltype(f)::value;
    if constexpr (tf4::kE4M3<FMT>) {
      if (multi(sh)) {
        if (v8) {
          const int64_t g = wave_grid(tf4::k_dequant8<FMT, tf4::SegN>, sh.nblocks, sh.be);
          launch_k(tf4::k_dequant8<FMT, tf4::SegN>, g, st, a, make_segn(sh));
        } else {
          const int64_t g = wave_grid(tf4::k_dequant<FMT, tf4::SegN>, sh.nblocks, sh.be);
          launch_k(tf4::k_dequant<FMT, tf4::SegN>, g, st, a, make_segn(sh));
        }
        return;
      }
    }
    if (v8) {
      const int64_t g = wave_grid(tf4::k_dequant8<FMT, tf4::Seg1>, sh.nblocks, sh.be);
      launch_k(tf4::k_dequant8<FMT, tf4::Seg1>, g, st, a, tf4::Seg1{});
    } else {
      const int64_t g = wave_grid(tf4::k_dequant<FMT, tf4::Seg1>, sh.nblocks, sh.be);
      launch_k(tf4::k_dequant<FMT, tf4::Seg1>, g, st, a, tf4::Seg1{});
    }
  });
  return launched();
}

tf4_status tf4_pack_guidance(const tf4_desc* desc, const uint8_t* codes, uint8_t* bits, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  if (!codes || !bits) return TF4_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(bits, 4)) return TF4_ERR_ALIGN;
  const int64_t units = sh.n / 32;
  const int tail = (sh.n % 32) != 0;
  const int64_t g = wave_grid(tf4::k_pack, units > 0 ? units : 1);
  launch_k(tf4::k_pack, g, reinterpret_cast<cudaStream_t>(stream), codes, bits, units, tail);
  return launched();
}

tf4_status tf4_unpack_guidance(const tf4_desc* desc, const uint8_t* bits, uint8_t* mant, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  if (!bits || !mant) return TF4_ERR_INVALID_ARG;
  if (!aligned(bits, 4) || !aligned(mant, 16)) return TF4_ERR_ALIGN;
  const int64_t units = sh.n / 16;  // rows*cols is a multiple of 16
  const int64_t g = wave_grid(tf4::k_unpack, units);
  launch_k(tf4::k_unpack, g, reinterpret_cast<cudaStream_t>(stream), bits, mant, units);
  return launched();
}

size_t tf4_blocked_scales_bytes(const tf4_desc* desc) {
  Shape sh;
  if (check_desc(desc, &sh) != TF4_OK) return 0;
  const int64_t nb = sh.cols / sh.be;
  return (size_t)((sh.rows + 127) / 128 * 128) * (size_t)((nb + 3) / 4 * 4);
}

tf4_status tf4_swizzle_scales(const tf4_desc* desc, const uint8_t* scales, uint8_t* blocked, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.n == 0) return TF4_OK;
  if (!scales || !blocked) return TF4_ERR_INVALID_ARG;
  if (!aligned(blocked, 16)) return TF4_ERR_ALIGN;
  const int64_t nb = sh.cols / sh.be;
  const int64_t ntc = (nb + 3) / 4;
  const int64_t nlines = (sh.rows + 127) / 128 * ntc * 32;  // 16-byte lines, 32 per tile
  const int64_t wave = (int64_t)sm_count() * occupancy(reinterpret_cast<const void*>(tf4::k_swizzle));
  const int64_t need = (nlines + kThreads - 1) / kThreads;
  launch_k(tf4::k_swizzle, need < wave ? need : wave, reinterpret_cast<cudaStream_t>(stream), scales, sh.rows, nb,
           ntc, nlines, reinterpret_cast<uint4*>(blocked));
  return launched();
}

tf4_status tf4_quantize_capture_noalloc(const tf4_desc* desc, const void* x, uint8_t* codes, uint8_t* scales,
                                        float* s_t, uint8_t* bits, int32_t* status, tf4_stream_t stream) {
  Shape sh;
  tf4_status e = check_desc(desc, &sh);
  if (e != TF4_OK) return e;
  if (sh.nseg > TF4_NOALLOC_MAX_SEGMENTS) return TF4_ERR_WORKSPACE;
  // The scratch array has one copy per device; the one used must be that of
  // the device the kernels run on, which is the current device, so a stream
  // of another device is refused.
  int cur = 0, sdev = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return TF4_ERR_CUDA;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cs == nullptr || cs == cudaStreamLegacy || cs == cudaStreamPerThread) {
    sdev = cur;  // the default streams belong to the current device
  } else if (cudaStreamGetDevice(cs, &sdev) != cudaSuccess) {
    cudaGetLastError();
    return TF4_ERR_INVALID_ARG;
  }
  if (sdev != cur) return TF4_ERR_INVALID_ARG;
  uint32_t* scratch = noalloc_scratch(cur);
  if (!scratch) return TF4_ERR_CUDA;
  // the amax pass uses num_segments + 1 words, the single-launch capture 3
  const size_t need = sizeof(uint32_t) * (size_t)(sh.nseg + 1 > 3 ? sh.nseg + 1 : 3);
  if (has_tensor_scale(sh.fmt) && sh.n > 0 &&
      cudaMemsetAsync(scratch, 0, need, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TF4_ERR_CUDA;
  return tf4_quantize_capture(desc, x, nullptr, codes, scales, s_t, bits, scratch, sizeof(tf4_noalloc_scratch),
                              status, stream);
}

tf4_status tf4_read_status(int32_t* dev_status, tf4_stream_t stream) {
  if (!dev_status) return TF4_ERR_INVALID_ARG;
  if (!aligned(dev_status, 4)) return TF4_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, dev_status, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return TF4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TF4_ERR_CUDA;
  if (cudaMemsetAsync(dev_status, 0, sizeof h, st) != cudaSuccess) return TF4_ERR_CUDA;
  if (h & TF4_DEV_NONFINITE) return TF4_ERR_NONFINITE;
  if (h & TF4_DEV_TIMEOUT) return TF4_ERR_TIMEOUT;
  return TF4_OK;
}

const char* tf4_status_string(tf4_status s) {
  switch (s) {
    case TF4_OK: return "ok";
    case TF4_ERR_INVALID_ARG: return "invalid argument";
    case TF4_ERR_SHAPE: return "invalid shape (rows/cols, or cols not a multiple of the block size)";
    case TF4_ERR_ALIGN: return "misaligned pointer";
    case TF4_ERR_WORKSPACE: return "workspace missing or too small";
    case TF4_ERR_NONFINITE: return "non-finite input";
    case TF4_ERR_TIMEOUT: return "a bounded device wait timed out";
    case TF4_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

int tf4_version(void) { return 2; }

int tf4_debug_bounds_enabled(void) {
#ifdef TF4_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

tf4_status tf4_debug_bounds_violations(uint64_t* count, tf4_stream_t stream) {
  if (!count) return TF4_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return TF4_ERR_CUDA;
  unsigned long long v = 0ull;
  if (cudaMemcpyFromSymbol(&v, tf4::g_tf4_bounds, sizeof v) != cudaSuccess) return TF4_ERR_CUDA;
  const unsigned long long zero = 0ull;
  if (cudaMemcpyToSymbol(tf4::g_tf4_bounds, &zero, sizeof zero) != cudaSuccess) return TF4_ERR_CUDA;
  *count = (uint64_t)v;
  return TF4_OK;
}

}  // extern "C"
