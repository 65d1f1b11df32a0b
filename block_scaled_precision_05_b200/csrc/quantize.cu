// quantize.cu -- bf16 -> NVFP4 / MXFP8 block quantization, global scales, and
// the diagnostic entry points.
//
// NVFP4 (hao-ai-lab-FastVideo nvfp4_config.py, module docstring: e2m1
// elements, group size 16, e4m3 scale per group, fp32 global scale,
// layout_128x4), per group of 16 along K:
//   amax = max|x|;  s = fl32(fl32(amax/6) * gs);  sfb = e4m3_rne_sat(s)
//   inv = sfb ? fl32(gs / value(sfb)) : 0;  code_i = e2m1_rne_sat(fl32(x_i*inv))
// MXFP8 (vllm-omni mxfp8_config.py, DiffusionMXFP8Config: 32 elements per
// float8_e8m0fnu scale, e4m3 elements, OCP MX), per group of 32:
//   e = clamp(floor(log2 amax) - 8, -127, 127);  sfb = e + 127;
//   q_i = e4m3_rne_sat(x_i * 2^-e)
// Scale bytes go straight to the 128x4 tile layout:
//   ((r/128)*(cols4/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4
//
// HBM-bound streaming kernels.  Fast paths (K % 64 == 0 for NVFP4, K % 128 ==
// 0 for MXFP8): one warp per row, one lane per group (16 or 32 elements read
// with adjacent 16-byte loads, so a warp step reads 1 or 2 KB of one row and
// the scale arithmetic is paid once per group), group amax in the integer
// domain (|bf16| bit patterns order like their values), hardware cvt with
// round-to-nearest-even and saturation, 8- or 32-byte code stores, and the four
// scale bytes of a 128x4 tile row gathered by shuffles into one 4-byte store.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "bsp_device.cuh"
#include "bsp_internal.h"
#include "norm_stats.cuh"

namespace bsp {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kUnroll = 2;  // warp steps in flight per row iteration
constexpr uint32_t kFull = 0xFFFFFFFFu;

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Input element formats (16-bit floats, two per 32-bit word, the element at
// the lower address in the low half).  In both, the bit pattern of |x| orders
// like its value.
struct InBf16 {
  using T2 = __nv_bfloat162;
  static constexpr uint32_t kInf = 0x7F80u, kMaxFinite = 0x7F7Fu;
  static __device__ __forceinline__ float value(uint32_t bits) { return __uint_as_float(bits << 16); }
  static __device__ __forceinline__ float2 values2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
  static __device__ __forceinline__ T2 abs2(uint32_t w) {
    T2 r;
    const uint32_t u = w & 0x7FFF7FFFu;
    memcpy(&r, &u, 4);
    return r;
  }
  static __device__ __forceinline__ uint32_t larger_half(T2 m) {
    const __nv_bfloat16 h = __hmax(__low2bfloat16(m), __high2bfloat16(m));
    uint16_t u;
    memcpy(&u, &h, 2);
    return u;
  }
};

struct InF16 {
  using T2 = __half2;
  static constexpr uint32_t kInf = 0x7C00u, kMaxFinite = 0x7BFFu;
  static __device__ __forceinline__ float value(uint32_t bits) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
  }
  static __device__ __forceinline__ float2 values2(uint32_t w) {
    __half2 h;
    memcpy(&h, &w, 4);
    return __half22float2(h);
  }
  static __device__ __forceinline__ T2 abs2(uint32_t w) {
    T2 r;
    const uint32_t u = w & 0x7FFF7FFFu;
    memcpy(&r, &u, 4);
    return r;
  }
  static __device__ __forceinline__ uint32_t larger_half(T2 m) {
    const __half h = __hmax(__low2half(m), __high2half(m));
    return __half_as_ushort(h);
  }
};

// |x| bit pattern for the tensor / row amax: NaN counts as 0 and +-inf as the
// largest finite value (x.abs().nan_to_num()).
template <class In>
__device__ __forceinline__ uint32_t sane_mag(uint32_t b16) {
  const uint32_t m = b16 & 0x7FFFu;
  if (m > In::kInf) return 0u;
  if (m == In::kInf) return In::kMaxFinite;
  return m;
}

// Packed maxima of |x| over the 8 elements of a 16-byte chunk, with the packed
// max instruction, which ignores a NaN operand.
template <class In>
__device__ __forceinline__ typename In::T2 absmax8_x2(const uint4& v) {
  return __hmax2(__hmax2(In::abs2(v.x), In::abs2(v.y)), __hmax2(In::abs2(v.z), In::abs2(v.w)));
}

// Bit pattern of the larger of two packed maxima; NaN elements are ignored (a
// group of NaNs only gives 0).
template <class In>
__device__ __forceinline__ uint32_t max_of_halves(typename In::T2 m) {
  const uint32_t u = In::larger_half(m);
  return u > In::kInf ? 0u : u;
}

// amax bit pattern of one 16-element group (two 16-byte chunks).
template <class In>
__device__ __forceinline__ uint32_t group_mag16(const uint4& a, const uint4& b) {
  return max_of_halves<In>(__hmax2(absmax8_x2<In>(a), absmax8_x2<In>(b)));
}

template <class In>
__device__ __forceinline__ uint32_t max_mag8(const uint4& v) {
  return max_of_halves<In>(absmax8_x2<In>(v));
}

// As max_mag8, with +-inf counted as the largest finite value (sane_mag).
template <class In>
__device__ __forceinline__ uint32_t max_sane_mag8(const uint4& v) {
  return min(max_mag8<In>(v), In::kMaxFinite);
}

__device__ __forceinline__ uint32_t warp_max(uint32_t m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
  return m;
}

// gs = amax > 0 ? fl32(2688 / amax) : 1, from a sanitized |x| bit pattern.
template <class In>
__device__ __forceinline__ float global_scale_from_mag(uint32_t mag) {
  return mag == 0u ? 1.0f : __fdiv_rn(2688.0f, In::value(mag));
}

// fl32(x / 6) for x a bf16 or fp16 magnitude: the product with fl32(1/6),
// corrected once by the fma residual r = x - 6q (a residual-corrected
// reciprocal product in the manner of Markstein's division: q' = q + r/6 with
// r exact by the fma).  For 0 and every positive finite bf16 and fp16 value
// this equals the correctly rounded quotient (checked exhaustively against
// exact rationals); +inf (the amax of a group holding an infinity) gives +inf.
__device__ __forceinline__ float div6_rn(float x) {
  constexpr float kSixth = 0x1.555556p-3f;  // fl32(1/6)
  const float q = __fmul_rn(x, kSixth);
  const float c = __fmaf_rn(__fmaf_rn(-q, 6.0f, x), kSixth, q);
  return x == __int_as_float(0x7F800000) ? x : c;
}

// fl32(gs / e4m3(b)) for every scale byte b (0 for b = 0): the decode factor
// of a per-tensor scale, built once per block so that a group looks it up
// instead of dividing.  Ends with a block barrier.  Used by the kernels whose
// time is instruction issue rather than DRAM (the fused RMSNorm ones and the
// short-row one); in the K % 64 streaming kernels it measured slower.
__device__ __forceinline__ void build_inv_table(float* tab, float gs) {
  for (uint32_t i = threadIdx.x; i < 256u; i += blockDim.x)
    tab[i] = i == 0u ? 0.0f : __fdiv_rn(gs, e4m3_pos_to_f32(i));
  __syncthreads();
}

// NVFP4 scale byte and reciprocal of one group with amax bit pattern `mag`
// (inv_tab: build_inv_table(gs), or NULL to divide).
template <class In>
__device__ __forceinline__ void nvfp4_scale(uint32_t mag, float gs, uint32_t& sfb, float& inv,
                                            const float* inv_tab = nullptr) {
  const float amax = In::value(mag);
  const float s = __fmul_rn(div6_rn(amax), gs);
  sfb = cvt_e4m3x2(s, 0.0f) & 0xFFu;
  inv = inv_tab ? inv_tab[sfb] : ((sfb == 0u) ? 0.0f : __fdiv_rn(gs, e4m3_pos_to_f32(sfb)));
}

// Decode factor fl32(gs / e4m3(b)) without a division per group.  A positive
// e4m3 value is an integer m in 1..15 times a power of two: m = 8 + f and
// 2^(E-10) for a normal byte (E, f), m = f and 2^-9 (the scale of E = 1) for
// a subnormal one.  Scaling by a power of two commutes with rounding while
// the result stays normal, so fl32(gs / e4m3(b)) = fl32(gs / m) * 2^(10 -
// max(E, 1)), with fl32(gs / m) taken from lane m of `quot` (quotient_lane).
// Normal here: gs >= 2688 / max finite > 2^-117 and e4m3(b) <= 480 keep every
// quotient and product at or above 2^-126; an overflow gives +inf in both
// forms.  All 32 lanes must take part (a warp shuffle).
__device__ __forceinline__ float quotient_lane(float gs) {
  const uint32_t m = lane_id();
  return (m == 0u || m > 15u) ? 0.0f : __fdiv_rn(gs, static_cast<float>(m));
}

__device__ __forceinline__ float inv_from_quotients(float quot, uint32_t sfb) {
  const uint32_t e = (sfb >> 3) & 0xFu, f = sfb & 7u;
  const float q = __shfl_sync(kFull, quot, e == 0u ? f : 8u + f);  // lane 0 holds 0: b = 0 gives 0
  const uint32_t e1 = e == 0u ? 1u : e;
  return __fmul_rn(q, __uint_as_float((137u - e1) << 23));
}

// NVFP4 scale byte and decode factor of one group from the row's quotients.
template <class In>
__device__ __forceinline__ void nvfp4_scale_q(uint32_t mag, float gs, float quot, uint32_t& sfb, float& inv) {
  const float s = __fmul_rn(div6_rn(In::value(mag)), gs);
  sfb = cvt_e4m3x2(s, 0.0f) & 0xFFu;
  inv = inv_from_quotients(quot, sfb);
}

// Eight elements (one 16-byte chunk) times inv -> eight e2m1 codes in one
// word.  The products are fp32 multiplies, two per packed instruction.
template <class In>
__device__ __forceinline__ uint32_t nvfp4_codes8(const uint4& v, float inv) {
  const float2 i2 = make_float2(inv, inv);
  const float2 p0 = mul2_rn(In::values2(v.x), i2), p1 = mul2_rn(In::values2(v.y), i2);
  const float2 p2 = mul2_rn(In::values2(v.z), i2), p3 = mul2_rn(In::values2(v.w), i2);
  return cvt_e2m1x8(p0.x, p0.y, p1.x, p1.y, p2.x, p2.y, p3.x, p3.y);
}

// Scale-factor tile layouts.  row_base(r, tiles) is the byte offset of the
// first of the four scale bytes (r, 4*tile_col .. +3) of tile column 0; tile
// column j is kTileBytes further.
//   128x4 (layout_128x4): 512-byte tiles of 128 rows x 4 columns, 32 lines of
//     16 bytes, line l holding rows l, l+32, l+64, l+96; what the tensor core
//     consumes.
//   8x4 (layout_8x4, the small-M layout of mm_fp4's use_8x4_sf_layout):
//     32-byte tiles of 8 rows x 4 columns, row-major.
struct Sf128x4 {
  static constexpr int kRowTile = 128, kTileBytes = 512;
  static __device__ __forceinline__ int64_t row_base(int64_t r, int64_t tiles) {
    return (r >> 7) * tiles * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4;
  }
};
struct Sf8x4 {
  static constexpr int kRowTile = 8, kTileBytes = 32;
  static __device__ __forceinline__ int64_t row_base(int64_t r, int64_t tiles) {
    return (r >> 3) * tiles * 32 + (r & 7) * 4;
  }
};

// Per-row encode scale of row r (warp-cooperative); lane 0 stores gs and 1/gs.
template <class In>
__device__ __forceinline__ float row_scale_pass(const uint16_t* __restrict__ row, int64_t K, int64_t r,
                                                float* row_gs, float* row_inv) {
  const uint32_t lane = lane_id();
  uint32_t m = 0;
  int64_t c = lane * 8;
  for (; c + 768 < K; c += 1024) {  // four independent 16-byte loads in flight
    const uint4 a = ldg16(row + c), b = ldg16(row + c + 256), d = ldg16(row + c + 512), e = ldg16(row + c + 768);
    m = max(max(m, max(max_sane_mag8<In>(a), max_sane_mag8<In>(b))), max(max_sane_mag8<In>(d), max_sane_mag8<In>(e)));
  }
  for (; c < K; c += 256) m = max(m, max_sane_mag8<In>(ldg16(row + c)));
  m = warp_max(m);
  const float gs = global_scale_from_mag<In>(m);
  if (lane == 0) {
    if (row_gs) row_gs[r] = gs;
    if (row_inv) row_inv[r] = __fdiv_rn(1.0f, gs);
  }
  return gs;
}

// ---------------------------------------------------------------------------
// NVFP4, K % 64 == 0.  Rows [M, Mp) are the scale padding (zeros).
// A "quad" is 64 elements = one 128x4 tile row = 8 lanes; a warp step is 4 quads.
// ---------------------------------------------------------------------------
// One lane quantizes one group of 16 (two adjacent 16-byte loads); a warp step
// covers 32 groups = 512 elements of one row.  U steps: 2U loads in flight per
// lane, then the quantization of each.  `lp`, `cp`, `sp` point at this lane's
// group, its 8 code bytes, and (for lanes with g % 4 == 0) its 4 scale bytes in
// the first step.
template <class In, class L, int U>
__device__ __forceinline__ void nvfp4_steps(const uint16_t* lp, uint8_t* cp, uint8_t* sp, bool live, float gs,
                                            bool store_sf, const float* inv_tab) {
  uint4 v[U][2];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    v[u][0] = live ? ldg16(lp + u * 512) : make_uint4(0u, 0u, 0u, 0u);
    v[u][1] = live ? ldg16(lp + u * 512 + 8) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    uint32_t sfb;
    float inv;
    nvfp4_scale<In>(group_mag16<In>(v[u][0], v[u][1]), gs, sfb, inv, inv_tab);
    uint2 w;
    w.x = nvfp4_codes8<In>(v[u][0], inv);
    w.y = nvfp4_codes8<In>(v[u][1], inv);
    const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
    const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
    const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
    if (live) *reinterpret_cast<uint2*>(cp + u * 256) = w;
    if (store_sf) *reinterpret_cast<uint32_t*>(sp + u * 8 * L::kTileBytes) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

// Per-tensor scale, short rows (K = 512 * S, S <= 3): a warp quantizes two rows
// per iteration with all 4S 16-byte loads of both rows issued up front, so the
// memory pipeline stays full although each row is only S warp steps long.
template <class In, class L, int S>
__global__ void __launch_bounds__(kQuantThreads, 3) nvfp4_quant_short_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t ld_x, const float* __restrict__ gs_ptr,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  constexpr int64_t K = 512 * S;
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float gs = __ldg(gs_ptr);
  const bool quad_lead = (lane & 3u) == 0u;
  __shared__ float inv_tab[256];
  build_inv_table(inv_tab, gs);
  for (int64_t r0 = 2 * warp; r0 < Mp; r0 += 2 * nwarps) {
    uint4 v[2][S][2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t r = r0 + h;
      const bool live = r < M;
      const uint16_t* lp = x + r * ld_x + lane * 16;
#pragma unroll
      for (int st = 0; st < S; ++st) {
        v[h][st][0] = live ? ldg16(lp + st * 512) : make_uint4(0u, 0u, 0u, 0u);
        v[h][st][1] = live ? ldg16(lp + st * 512 + 8) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t r = r0 + h;
      if (r >= Mp) break;
      const bool live = r < M;
      uint8_t* cp = codes + r * (K >> 1) + lane * 8;
      uint8_t* sp = sf + L::row_base(r, K >> 6) + (lane >> 2) * L::kTileBytes;
#pragma unroll
      for (int st = 0; st < S; ++st) {
        uint32_t sfb;
        float inv;
        nvfp4_scale<In>(group_mag16<In>(v[h][st][0], v[h][st][1]), gs, sfb, inv, inv_tab);
        uint2 w;
        w.x = nvfp4_codes8<In>(v[h][st][0], inv);
        w.y = nvfp4_codes8<In>(v[h][st][1], inv);
        const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
        const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
        const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
        if (live) *reinterpret_cast<uint2*>(cp + st * 256) = w;
        if (quad_lead)
          *reinterpret_cast<uint32_t*>(sp + st * 8 * L::kTileBytes) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
    }
  }
}

// Per-row (per-token) scale, K % 64 == 0 and K <= 16 * 256 * kRowG: one block
// of 256 threads per row.  Thread t holds groups t, t+256, ... of the row in
// registers (two adjacent 16-byte loads each, all issued at once), the row
// amax is reduced through shared memory, and the row is quantized from the
// registers, so each row costs one memory round trip.
constexpr int kRowG = 4;

template <class In, class L>
__global__ void __launch_bounds__(kQuantThreads) nvfp4_quant_rowblock_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t K, int64_t ld_x, float* __restrict__ row_gs,
    float* __restrict__ row_inv, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  __shared__ uint32_t red[kQuantThreads / 32];
  __shared__ float gs_sh;
  const uint32_t lane = lane_id();
  const int t = static_cast<int>(threadIdx.x);
  const int groups = static_cast<int>(K >> 4);
  const int64_t tiles_per_band = groups >> 2;
  for (int64_t r = blockIdx.x; r < Mp; r += gridDim.x) {
    const bool live = r < M;
    const uint16_t* row = x + r * ld_x;
    uint4 v[kRowG][2];
    uint32_t mag = 0;
#pragma unroll
    for (int i = 0; i < kRowG; ++i) {
      const int g = t + i * kQuantThreads;
      const bool in = live && g < groups;
      v[i][0] = in ? ldg16(row + g * 16) : make_uint4(0u, 0u, 0u, 0u);
      v[i][1] = in ? ldg16(row + g * 16 + 8) : make_uint4(0u, 0u, 0u, 0u);
      mag = max(mag, max(max_sane_mag8<In>(v[i][0]), max_sane_mag8<In>(v[i][1])));
    }
    mag = warp_max(mag);
    if (lane == 0) red[threadIdx.x >> 5] = mag;
    __syncthreads();
    if (threadIdx.x < 32) {
      uint32_t m = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0u;
      m = warp_max(m);
      if (threadIdx.x == 0) {
        const float gs = global_scale_from_mag<In>(m);
        gs_sh = gs;
        if (live) {
          if (row_gs) row_gs[r] = gs;
          if (row_inv) row_inv[r] = __fdiv_rn(1.0f, gs);
        }
      }
    }
    __syncthreads();
    const float gs = gs_sh;
    uint8_t* crow = codes + r * (K >> 1);
    const int64_t sbase = L::row_base(r, tiles_per_band);
#pragma unroll
    for (int i = 0; i < kRowG; ++i) {
      const int g = t + i * kQuantThreads;
      // within a warp, groups are consecutive, so lanes 4j..4j+3 own one scale word
      if (i * kQuantThreads + (t & ~31) >= groups) break;  // warp-uniform
      uint32_t sfb;
      float inv;
      nvfp4_scale<In>(group_mag16<In>(v[i][0], v[i][1]), gs, sfb, inv);
      uint2 w;
      w.x = nvfp4_codes8<In>(v[i][0], inv);
      w.y = nvfp4_codes8<In>(v[i][1], inv);
      const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
      const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
      const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
      if (g < groups) {
        if (live) *reinterpret_cast<uint2*>(crow + g * 8) = w;
        if ((g & 3) == 0)
          *reinterpret_cast<uint32_t*>(sf + sbase + (g >> 2) * L::kTileBytes) =
              sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
    }
    __syncthreads();  // red / gs_sh are reused by the next row
  }
}

// Per-row (per-token) scale, K = 512 * S * G (hidden sizes 1024, 1536, 2048,
// 5120): each row by S warps whose threads hold it in registers (thread t of
// the row's S * 32 owns groups t, t + 32 S, ... : 2G 16-byte loads, all
// issued at once), the row amax by warp reductions and, for S > 1, a named
// barrier over the row's warps, then the row quantized from the registers --
// one DRAM round trip per row.  A block holds blockDim / (32 S) such row
// teams.  S trades the serial work of one thread (G groups) against barrier
// and reduction cost: few rows take large S, many rows S = 1.  Rows [M, Mp)
// write their zero scale bytes only.
constexpr int kRowTeamMax = 8;  // row teams per block at most

template <class In, class L, int G, int S>
__global__ void __launch_bounds__(kQuantThreads) nvfp4_quant_rowreg_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t ld_x, float* __restrict__ row_gs,
    float* __restrict__ row_inv, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  constexpr int64_t K = 512 * S * G;
  constexpr int kTeam = 32 * S;
  __shared__ uint32_t red[2][kRowTeamMax][S];
  const uint32_t lane = lane_id();
  const int team = static_cast<int>(threadIdx.x) / kTeam;
  const int t = static_cast<int>(threadIdx.x) % kTeam;
  const int teams = static_cast<int>(blockDim.x) / kTeam;
  const bool quad_lead = (lane & 3u) == 0u;
  int parity = 0;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * teams + team; r < Mp;
       r += static_cast<int64_t>(gridDim.x) * teams, parity ^= 1) {
    const bool live = r < M;
    const uint16_t* lp = x + r * ld_x + t * 16;
    uint4 v[G][2];
#pragma unroll
    for (int i = 0; i < G; ++i) {
      v[i][0] = live ? ldg16(lp + i * 16 * kTeam) : make_uint4(0u, 0u, 0u, 0u);
      v[i][1] = live ? ldg16(lp + i * 16 * kTeam + 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    // group amaxes, kept for the scales; the row amax is their maximum with
    // +-inf counted as the largest finite value (NaN-ignoring maxima compose)
    uint32_t gm[G], mag = 0;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      gm[i] = group_mag16<In>(v[i][0], v[i][1]);
      mag = max(mag, gm[i]);
    }
    mag = min(warp_max(mag), In::kMaxFinite);
    if constexpr (S > 1) {
      // the team's warps meet at named barrier 1 + team; red alternates by
      // row parity, so one barrier per row orders writes against old reads
      if (lane == 0) red[parity][team][t >> 5] = mag;
      asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(kTeam) : "memory");
#pragma unroll
      for (int w = 0; w < S; ++w) mag = max(mag, red[parity][team][w]);
    }
    const float gs = global_scale_from_mag<In>(mag);
    if (live && t == 0) {
      if (row_gs) row_gs[r] = gs;
      if (row_inv) row_inv[r] = __fdiv_rn(1.0f, gs);
    }
    const float quot = quotient_lane(gs);
    uint8_t* cp = codes + r * (K >> 1) + t * 8;
    uint8_t* sp = sf + L::row_base(r, K >> 6) + (t >> 2) * L::kTileBytes;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      uint32_t sfb;
      float inv;
      nvfp4_scale_q<In>(gm[i], gs, quot, sfb, inv);
      uint2 w;
      w.x = nvfp4_codes8<In>(v[i][0], inv);
      w.y = nvfp4_codes8<In>(v[i][1], inv);
      const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
      const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
      const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
      if (live) *reinterpret_cast<uint2*>(cp + i * 8 * kTeam) = w;
      if (quad_lead)
        *reinterpret_cast<uint32_t*>(sp + i * (kTeam / 4) * L::kTileBytes) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
    }
  }
}

// Row r (K % 64 == 0) with scale gs, by one warp: group g = 32 * step + lane
// covers elements 16 g, code bytes 8 g and scale tile g / 4.  A row past the
// tensor (live false) only writes its zero scale bytes.
template <class In, class L, int U = kUnroll>
__device__ __forceinline__ void nvfp4_row_k64(const uint16_t* row, int64_t K, int64_t r, bool live, float gs,
                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf, uint32_t lane,
                                              const float* inv_tab) {
  const int64_t groups = K >> 4;
  const int64_t steps = groups >> 5;  // full warp steps (32 groups) per row
  const int64_t rem = groups & 31;    // groups of a last, partial step (a multiple of 4)
  const bool quad_lead = (lane & 3u) == 0u;
  const uint16_t* lp = row + lane * 16;
  uint8_t* cp = codes + r * (K >> 1) + lane * 8;
  uint8_t* sp = sf + L::row_base(r, groups >> 2) + (lane >> 2) * L::kTileBytes;
  constexpr int kStepSf = 8 * L::kTileBytes;  // a warp step covers 8 scale tiles
  int64_t st = 0;
  for (; st + U <= steps; st += U)
    nvfp4_steps<In, L, U>(lp + st * 512, cp + st * 256, sp + st * kStepSf, live, gs, quad_lead, inv_tab);
  for (; st < steps; ++st)
    nvfp4_steps<In, L, 1>(lp + st * 512, cp + st * 256, sp + st * kStepSf, live, gs, quad_lead, inv_tab);
  if (rem) {
    const bool in = lane < rem;  // groups beyond the row end are predicated off
    nvfp4_steps<In, L, 1>(in ? lp + st * 512 : lp, in ? cp + st * 256 : cp, in ? sp + st * kStepSf : sp, live && in,
                          gs, in && quad_lead, inv_tab);
  }
}

template <class In, class L, bool kPerRow>
__global__ void __launch_bounds__(kQuantThreads) nvfp4_quant_k64_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t K, int64_t ld_x, const float* __restrict__ gs_ptr,
    float* __restrict__ row_gs, float* __restrict__ row_inv, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float gs_tensor = kPerRow ? 1.0f : __ldg(gs_ptr);

  for (int64_t r = warp; r < Mp; r += nwarps) {
    const bool live = r < M;
    const uint16_t* row = x + r * ld_x;
    float gs = gs_tensor;
    if (kPerRow && live) gs = row_scale_pass<In>(row, K, r, row_gs, row_inv);
    nvfp4_row_k64<In, L>(row, K, r, live, gs, codes, sf, lane, nullptr);
  }
}

// ---------------------------------------------------------------------------
// NVFP4, any K % 16 == 0: one warp per row, one lane per group of 16.
// ---------------------------------------------------------------------------
template <class In, class L, bool kPerRow>
__global__ void __launch_bounds__(kQuantThreads) nvfp4_quant_generic_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t K, int64_t ld_x, const float* __restrict__ gs_ptr,
    float* __restrict__ row_gs, float* __restrict__ row_inv, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  const uint32_t lane = lane_id();
  const int64_t groups = K >> 4, cols4 = (groups + 3) & ~int64_t(3);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float gs_tensor = kPerRow ? 1.0f : __ldg(gs_ptr);

  for (int64_t r = warp; r < Mp; r += nwarps) {
    const bool live = r < M;
    const uint16_t* row = x + r * ld_x;
    float gs = gs_tensor;
    if (kPerRow && live) gs = row_scale_pass<In>(row, K, r, row_gs, row_inv);
    const int64_t sfb_row = L::row_base(r, cols4 >> 2);
    for (int64_t c = lane; c < cols4; c += 32) {
      uint32_t sfb = 0;
      if (live && c < groups) {
        const uint4 a = ldg16(row + c * 16), b = ldg16(row + c * 16 + 8);
        float inv;
        nvfp4_scale<In>(group_mag16<In>(a, b), gs, sfb, inv);
        uint2 w;
        w.x = nvfp4_codes8<In>(a, inv);
        w.y = nvfp4_codes8<In>(b, inv);
        *reinterpret_cast<uint2*>(codes + r * (K >> 1) + c * 8) = w;
      }
      sf[sfb_row + (c >> 2) * L::kTileBytes + (c & 3)] = static_cast<uint8_t>(sfb);
    }
  }
}

// ---------------------------------------------------------------------------
// Norms fused into the NVFP4 quantizer (the producer of a pre-quantized
// activation: hao-ai-lab-FastVideo nvfp4_config.py, NVFP4QuantizeMethod.apply
// with `pre_quantized` from a fused norm+quant call).  Per row:
//   RMSNorm   ms = mean(x^2), rstd = fl32(1 / sqrt(fl32(ms + eps)))
//             y_k = bf16(fl32(fl32(x_k * rstd) * gamma_k))
//   LayerNorm mean, var = the row's mean and population variance,
//             rstd = fl32(1 / sqrt(fl32(var + eps)))
//             y_k = bf16(fl32(fl32(fl32(fl32(x_k - mean) * rstd) * gamma_k) + beta_k))
//             (gamma 1 and beta -0 when absent: both are exact identities)
// with the statistics the exact values rounded once to fp32 (norm_stats.cuh),
// and rstd correctly rounded.  y is then quantized exactly as nvfp4_quantize
// quantizes a bf16 input, so the result equals the norm to bf16 followed by
// nvfp4_quantize, without writing y.  One warp per row.
// ---------------------------------------------------------------------------
constexpr int kNormWarps = kQuantThreads / 32;
constexpr uint32_t kBf16OnePair = 0x3F803F80u, kBf16NegZeroPair = 0x80008000u;

// Eight normalised outputs as bf16 pairs (RMSNorm), gamma as fp32 pairs.
__device__ __forceinline__ uint4 rmsnorm8(const uint4& xv, const float2 (&g)[4], float rstd) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const float2 r2 = make_float2(rstd, rstd);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // two fp32 products per packed instruction, each rounded as a scalar one
    const float2 y = mul2_rn(mul2_rn(InBf16::values2(xw[i]), r2), g[i]);
    const __nv_bfloat162 h = __floats2bfloat162_rn(y.x, y.y);
    memcpy(&o[i], &h, 4);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight normalised outputs as bf16 pairs (LayerNorm), gamma and beta as fp32 pairs.
__device__ __forceinline__ uint4 layernorm8(const uint4& xv, const float2 (&g)[4], const float2 (&b)[4], float mean,
                                            float rstd) {
  const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
  const float2 nm2 = make_float2(-mean, -mean), r2 = make_float2(rstd, rstd);
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 d = add2_rn(InBf16::values2(xw[i]), nm2);  // x - mean, rounded once
    const float2 t = mul2_rn(mul2_rn(d, r2), g[i]);
    // the shift as scalar adds: a packed add right after a packed multiply has
    // been seen fused into one multiply-add (one rounding instead of two), even
    // with contraction switched off for this file
    const float2 y = make_float2(__fadd_rn(t.x, b[i].x), __fadd_rn(t.y, b[i].y));
    const __nv_bfloat162 h = __floats2bfloat162_rn(y.x, y.y);
    memcpy(&o[i], &h, 4);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Eight bf16 values as fp32 pairs (exact).
struct Pairs8 {
  float2 v[4];
  __device__ __forceinline__ explicit Pairs8(const uint4& w)
      : v{InBf16::values2(w.x), InBf16::values2(w.y), InBf16::values2(w.z), InBf16::values2(w.w)} {}
  __device__ __forceinline__ Pairs8(const float4& a, const float4& b)
      : v{make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y), make_float2(b.z, b.w)} {}
};

// The per-row parameters of either norm and its elementwise map.
struct NormRow {
  float mean;  // LayerNorm only
  float rstd;
};

template <bool kLN>
__device__ __forceinline__ uint4 norm8(const uint4& xv, const Pairs8& g, const Pairs8& b, const NormRow& p) {
  if constexpr (kLN)
    return layernorm8(xv, g.v, b.v, p.mean, p.rstd);
  else
    return rmsnorm8(xv, g.v, p.rstd);
}

// Exact row statistics from the row in global memory (the rare path; the row
// is re-read): ms, or mean and var.
template <bool kLN>
__device__ __noinline__ void norm_row_exact(const uint16_t* __restrict__ row, int64_t K,
                                            normstats::ExactSums* xs, float* a, float* b) {
  const uint32_t lane = lane_id();
  normstats::exact_clear(xs);
  for (int64_t g = lane; g < (K >> 4); g += 32) {
    normstats::exact_add8(xs, ldg16(row + g * 16), kLN);
    normstats::exact_add8(xs, ldg16(row + g * 16 + 8), kLN);
  }
  __syncwarp();
  float ea = 0.0f, eb = 0.0f;
  if (lane == 0) {
    if constexpr (kLN)
      normstats::exact_mean_var(xs, static_cast<uint32_t>(K), &ea, &eb);
    else
      ea = normstats::exact_ms(xs, static_cast<uint32_t>(K));
  }
  *a = __shfl_sync(kFull, ea, 0);
  *b = __shfl_sync(kFull, eb, 0);
  __syncwarp();
}

// A LayerNorm row whose fast bounds left the statistics open: the mean
// decided exactly from the fp64 sum when that sum is provably exact (the
// row's smallest nonzero |x| is re-read), and the variance from its bound.
__device__ __noinline__ bool ln_row_mean_exact(const uint16_t* __restrict__ row, int64_t K, double s1, double s2,
                                               double rK, float* mean, float* var) {
  uint32_t m = 0xFFFFFFFFu;
  for (int64_t g = lane_id(); g < (K >> 4); g += 32) {
    m = normstats::min_nonzero_mag8(ldg16(row + g * 16), m);
    m = normstats::min_nonzero_mag8(ldg16(row + g * 16 + 8), m);
  }
  m = __reduce_min_sync(kFull, min(m & 0xFFFFu, m >> 16));
  if (!normstats::ln_var_fast(s1, s2, K, rK, var)) return false;
  return normstats::ln_mean_exact(s1, s2, K, rK, m, mean);
}

// Row statistics.  `each(f)` applies f to each of this lane's 16-byte chunks
// of the row (any order; the chunks of the 32 lanes cover the row once);
// `row` is the row in global memory, re-read by the exact path.
template <bool kLN, class Each>
__device__ __forceinline__ NormRow norm_row_stats(Each each, const uint16_t* row, int64_t K, double rK, float eps,
                                                  normstats::ExactSums* xs) {
  NormRow p;
  if constexpr (!kLN) {
    double acc = 0.0;
    each([&](const uint4& v) { acc = normstats::sumsq8(v, acc); });
    acc = normstats::warp_sum(acc);
    float ms, unused;
    if (!normstats::ms_fast(acc, K, rK, &ms)) norm_row_exact<false>(row, K, xs, &ms, &unused);  // warp-uniform
    p.mean = 0.0f;
    p.rstd = __frsqrt_rn(__fadd_rn(ms, eps));
  } else {
    double s1 = 0.0, s2 = 0.0;
    each([&](const uint4& v) { normstats::sums8(v, s1, s2); });
    s1 = normstats::warp_sum(s1);
    s2 = normstats::warp_sum(s2);
    float mean, var;
    if (!normstats::ln_fast(s1, s2, K, rK, &mean, &var) &&  // warp-uniform
        !ln_row_mean_exact(row, K, s1, s2, rK, &mean, &var))
      norm_row_exact<true>(row, K, xs, &mean, &var);
    p.mean = mean;
    p.rstd = __frsqrt_rn(__fadd_rn(var, eps));
  }
  return p;
}

__device__ __forceinline__ uint4 ldg16_or(const uint16_t* p, uint32_t fill) {
  return p ? ldg16(p) : make_uint4(fill, fill, fill, fill);
}

// gamma (and beta) as fp32 in the dynamic shared memory of a block of the
// general norm kernel: float4 [((g >> 5) * 4 + 2 half + j) * 32 + (g & 31)]
// holds elements [16 g + 8 half + 4 j, +4), so that the 32 lanes of a warp
// (groups g = lane + 32 i) read one contiguous 512-byte line per 16-byte load;
// beta follows gamma.  Used while both fit in kNormStageMaxBytes: on a
// 32760 x 5120 activation (the Wan-14B hidden size) staging took RMSNorm from 113 to 110 us and LayerNorm
// from 177 to 170 us (20 and 40 KB a block), but 54 KB at K = 13824 (RMSNorm)
// made it 17% slower, the shared memory taking L1 from the row re-reads.
constexpr size_t kNormStageMaxBytes = 40 * 1024;
static_assert(kNormStageMaxBytes + 4096 <= 48 * 1024, "staged bytes + static shared memory within the default limit");
__host__ __device__ constexpr int64_t norm_stage_quads(int64_t K) { return ((K >> 4) + 31) / 32 * 128; }
inline size_t norm_stage_bytes(int64_t K, bool ln) {
  return static_cast<size_t>(norm_stage_quads(K)) * sizeof(float4) * (ln ? 2 : 1);
}

// Any K % 16 == 0: the statistics pass(es), then (per-token scales) the row
// amax of y, then the groups; the later passes re-read the row from cache.
// kStaged: gamma and beta from shared memory as fp32 (converted once per
// block), else re-read as bf16 for every row.
template <class L, bool kPerRow, bool kLN, bool kStaged>
__global__ void __launch_bounds__(kQuantThreads) nvfp4_norm_quant_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t K, int64_t ld_x, const uint16_t* __restrict__ gamma,
    const uint16_t* __restrict__ beta, float eps, const float* __restrict__ gs_ptr, float* __restrict__ row_gs,
    float* __restrict__ row_inv, float* __restrict__ row_mean, float* __restrict__ row_rstd,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  const uint32_t lane = lane_id();
  const int64_t groups = K >> 4, cols4 = (groups + 3) & ~int64_t(3);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float gs_tensor = kPerRow ? 1.0f : __ldg(gs_ptr);
  const double rK = 1.0 / static_cast<double>(K);
  __shared__ float inv_tab[256];
  __shared__ normstats::ExactSums xsum[kNormWarps];
  if constexpr (!kPerRow) build_inv_table(inv_tab, gs_tensor);
  normstats::ExactSums* xs = &xsum[threadIdx.x >> 5];
  const uint16_t* bt = kLN ? beta : nullptr;
  extern __shared__ float4 aff[];  // kStaged: gamma, then beta
  const int64_t nq = norm_stage_quads(K);
  if constexpr (kStaged) {
    for (int64_t i = threadIdx.x; i < nq; i += blockDim.x) {
      const int64_t g = (i >> 7) * 32 + (i & 31);
      const int64_t c = g * 16 + ((i >> 6) & 1) * 8 + ((i >> 5) & 1) * 4;
      auto quad = [&](const uint16_t* t, float fill) {
        if (!t || g >= groups) return make_float4(fill, fill, fill, fill);
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(t + c));
        const float2 a = InBf16::values2(w.x), b = InBf16::values2(w.y);
        return make_float4(a.x, a.y, b.x, b.y);
      };
      aff[i] = quad(gamma, 1.0f);
      if constexpr (kLN) aff[nq + i] = quad(bt, -0.0f);
    }
    __syncthreads();
  }

  for (int64_t r = warp; r < Mp; r += nwarps) {
    const int64_t sfb_row = L::row_base(r, cols4 >> 2);
    if (r >= M) {  // scale padding rows
      for (int64_t c = lane; c < cols4; c += 32) sf[sfb_row + (c >> 2) * L::kTileBytes + (c & 3)] = 0;
      continue;
    }
    const uint16_t* row = x + r * ld_x;
    auto each = [&](auto f) {
      for (int64_t g = lane; g < groups; g += 32) {
        f(ldg16(row + g * 16));
        f(ldg16(row + g * 16 + 8));
      }
    };
    const NormRow p = norm_row_stats<kLN>(each, row, K, rK, eps, xs);
    if (lane == 0) {
      if (row_rstd) row_rstd[r] = p.rstd;
      if (kLN && row_mean) row_mean[r] = p.mean;
    }
    auto y8 = [&](int64_t c) {  // normalised elements [c, c + 8) as bf16 pairs
      if constexpr (kStaged) {
        const int64_t g = c >> 4;
        const int64_t q = ((g >> 5) * 4 + ((c >> 3) & 1) * 2) * 32 + (g & 31);
        const Pairs8 gp(aff[q], aff[q + 32]);
        return norm8<kLN>(ldg16(row + c), gp, kLN ? Pairs8(aff[nq + q], aff[nq + q + 32]) : gp, p);
      } else {
        return norm8<kLN>(ldg16(row + c), Pairs8(ldg16_or(gamma ? gamma + c : nullptr, kBf16OnePair)),
                          Pairs8(ldg16_or(bt ? bt + c : nullptr, kBf16NegZeroPair)), p);
      }
    };
    float gs = gs_tensor, quot = 0.0f;
    if (kPerRow) {
      uint32_t mag = 0;
      for (int64_t g = lane; g < groups; g += 32)
        mag = max(mag, max(max_sane_mag8<InBf16>(y8(g * 16)), max_sane_mag8<InBf16>(y8(g * 16 + 8))));
      mag = warp_max(mag);
      gs = global_scale_from_mag<InBf16>(mag);
      quot = quotient_lane(gs);
      if (lane == 0) {
        if (row_gs) row_gs[r] = gs;
        if (row_inv) row_inv[r] = __fdiv_rn(1.0f, gs);
      }
    }
    // warp-uniform trip count: the per-token decode factor takes a shuffle
    for (int64_t c0 = 0; c0 < cols4; c0 += 32) {
      const int64_t c = c0 + lane;
      uint32_t sfb = 0;
      if constexpr (kPerRow) {
        const bool in = c < groups;
        const uint4 y0 = in ? y8(c * 16) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 y1 = in ? y8(c * 16 + 8) : make_uint4(0u, 0u, 0u, 0u);
        float inv;
        nvfp4_scale_q<InBf16>(group_mag16<InBf16>(y0, y1), gs, quot, sfb, inv);  // all lanes
        if (in) {
          uint2 w;
          w.x = nvfp4_codes8<InBf16>(y0, inv);
          w.y = nvfp4_codes8<InBf16>(y1, inv);
          *reinterpret_cast<uint2*>(codes + r * (K >> 1) + c * 8) = w;
        } else {
          sfb = 0;  // scale padding columns
        }
      } else if (c < groups) {
        const uint4 y0 = y8(c * 16), y1 = y8(c * 16 + 8);
        float inv;
        nvfp4_scale<InBf16>(group_mag16<InBf16>(y0, y1), gs, sfb, inv, inv_tab);
        uint2 w;
        w.x = nvfp4_codes8<InBf16>(y0, inv);
        w.y = nvfp4_codes8<InBf16>(y1, inv);
        *reinterpret_cast<uint2*>(codes + r * (K >> 1) + c * 8) = w;
      }
      if (c < cols4) sf[sfb_row + (c >> 2) * L::kTileBytes + (c & 3)] = static_cast<uint8_t>(sfb);
    }
  }
}

// K = 512 * S (S = 3, 4: the Wan-1.3B hidden size 1536 among them): the same
// arithmetic with every row read from DRAM once and kept in registers.  Lane
// l holds elements [512 s + 16 l, 512 s + 16 l + 16) of the row for s < S (one
// group of 16 per slab); gamma (and beta) are converted to fp32 once per block
// into shared memory, in the order the lanes read them.  A warp loads R rows
// before working on the first, like
// nvfp4_quant_short_kernel.  Rows [M, Mp) are scale padding: y = 0, so their
// scale bytes are 0.
#ifndef BSP_RMSNORM_ROWS
#define BSP_RMSNORM_ROWS 1  // rows in flight per warp at K = 1536
#endif
#ifndef BSP_RMSNORM_MIN_BLOCKS
#define BSP_RMSNORM_MIN_BLOCKS 3  // resident blocks per SM the K = 1536 kernel is compiled for
#endif
template <bool kPerRow, bool kLN, int S, int R, int kMinBlocks>
__global__ void __launch_bounds__(kQuantThreads, kMinBlocks) nvfp4_norm_quant_short_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t Mp, int64_t ld_x, const uint16_t* __restrict__ gamma,
    const uint16_t* __restrict__ beta, float eps, const float* __restrict__ gs_ptr, float* __restrict__ row_gs,
    float* __restrict__ row_inv, float* __restrict__ row_mean, float* __restrict__ row_rstd,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  using L = Sf128x4;
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  constexpr int64_t K = 512 * S;
  const uint32_t lane = lane_id();
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const float gs_tensor = kPerRow ? 1.0f : __ldg(gs_ptr);
  constexpr double rK = 1.0 / static_cast<double>(K);
  __shared__ float inv_tab[256];
  __shared__ normstats::ExactSums xsum[kNormWarps];
  if constexpr (!kPerRow) build_inv_table(inv_tab, gs_tensor);
  normstats::ExactSums* xs = &xsum[threadIdx.x >> 5];
  const bool quad_lead = (lane & 3u) == 0u;
  // float4 [((s * 2 + half) * 2 + j) * 32 + l] holds elements [512 s + 16 l +
  // 8 half + 4 j, +4) of gamma (beta): for fixed (s, half, j) the 32 lanes read
  // one contiguous 512-byte line.  Absent: gamma 1, beta -0 (exact identities).
  constexpr int kQuads = S * 128;
  __shared__ float4 g_s[kQuads];
  __shared__ float4 b_s[kLN ? kQuads : 1];
  for (int i = threadIdx.x; i < kQuads; i += blockDim.x) {
    const int c = (i >> 7) * 512 + (i & 31) * 16 + ((i >> 6) & 1) * 8 + ((i >> 5) & 1) * 4;
    auto quad = [&](const uint16_t* t, float fill) {
      if (!t) return make_float4(fill, fill, fill, fill);
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(t + c));
      const float2 a = InBf16::values2(w.x), b = InBf16::values2(w.y);
      return make_float4(a.x, a.y, b.x, b.y);
    };
    g_s[i] = quad(gamma, 1.0f);
    if constexpr (kLN) b_s[i] = quad(beta, -0.0f);
  }
  __syncthreads();
  for (int64_t r0 = R * warp; r0 < Mp; r0 += R * nwarps) {
    uint4 v[R][S][2];
#pragma unroll
    for (int h = 0; h < R; ++h) {
      const int64_t r = r0 + h;
      const bool live = r < M;
      const uint16_t* lp = x + r * ld_x + lane * 16;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        v[h][s][0] = live ? ldg16(lp + s * 512) : make_uint4(0u, 0u, 0u, 0u);
        v[h][s][1] = live ? ldg16(lp + s * 512 + 8) : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int h = 0; h < R; ++h) {
      const int64_t r = r0 + h;
      if (r >= Mp) break;
      const bool live = r < M;
      NormRow p{0.0f, 0.0f};
      if (live) {  // warp-uniform
        auto each = [&](auto f) {
#pragma unroll
          for (int s = 0; s < S; ++s) {
            f(v[h][s][0]);
            f(v[h][s][1]);
          }
        };
        p = norm_row_stats<kLN>(each, x + r * ld_x, K, rK, eps, xs);
        if (lane == 0) {
          if (row_rstd) row_rstd[r] = p.rstd;
          if (kLN && row_mean) row_mean[r] = p.mean;
        }
      }
      // y is recomputed where it is needed rather than held (register pressure)
      auto y8 = [&](int s, int half) {
        const int q = (s * 2 + half) * 64 + static_cast<int>(lane);
        if constexpr (kLN)
          return norm8<kLN>(v[h][s][half], Pairs8(g_s[q], g_s[q + 32]), Pairs8(b_s[q], b_s[q + 32]), p);
        else
          return norm8<kLN>(v[h][s][half], Pairs8(g_s[q], g_s[q + 32]), Pairs8(g_s[q], g_s[q + 32]), p);
      };
      float gs = gs_tensor, quot = 0.0f;
      uint32_t gm[S];  // per-token: the group amaxes of y, kept for the scales
      if (kPerRow) {
        uint32_t mag = 0;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          gm[s] = group_mag16<InBf16>(y8(s, 0), y8(s, 1));
          mag = max(mag, gm[s]);
        }
        mag = min(warp_max(mag), InBf16::kMaxFinite);
        gs = global_scale_from_mag<InBf16>(mag);
        quot = quotient_lane(gs);
        if (live && lane == 0) {
          if (row_gs) row_gs[r] = gs;
          if (row_inv) row_inv[r] = __fdiv_rn(1.0f, gs);
        }
      }
      uint8_t* cp = codes + r * (K >> 1) + lane * 8;
      uint8_t* sp = sf + L::row_base(r, K >> 6) + (lane >> 2) * L::kTileBytes;
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const uint4 y0 = y8(s, 0), y1 = y8(s, 1);
        uint32_t sfb;
        float inv;
        if constexpr (kPerRow)
          nvfp4_scale_q<InBf16>(gm[s], gs, quot, sfb, inv);
        else
          nvfp4_scale<InBf16>(group_mag16<InBf16>(y0, y1), gs, sfb, inv, inv_tab);
        uint2 w;
        w.x = nvfp4_codes8<InBf16>(y0, inv);
        w.y = nvfp4_codes8<InBf16>(y1, inv);
        if (!live) sfb = 0u;  // scale padding (LayerNorm's beta would make y nonzero there)
        const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
        const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
        const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
        if (live) *reinterpret_cast<uint2*>(cp + s * 256) = w;
        if (quad_lead)
          *reinterpret_cast<uint32_t*>(sp + s * 8 * L::kTileBytes) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
    }
  }
}

// Row statistics alone (diagnostic entry bsp_debug_norm_stats): per row the
// RMSNorm ms, or the LayerNorm mean and var, each as the fast decision with its
// exact fallbacks (exact_only = false) or always from the exact sums; path[r]
// = 0 where the fp64 bounds decided, 2 where the LayerNorm mean came from a
// provably exact fp64 sum, 1 where the exact integer sums were used.
template <bool kLN>
__global__ void __launch_bounds__(kQuantThreads) norm_stats_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                    int64_t K, int64_t ld_x, bool exact_only,
                                                                    float* __restrict__ stat0,
                                                                    float* __restrict__ stat1, int* __restrict__ path) {
  const uint32_t lane = lane_id();
  const int64_t groups = K >> 4;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const double rK = 1.0 / static_cast<double>(K);
  __shared__ normstats::ExactSums xsum[kNormWarps];
  normstats::ExactSums* xs = &xsum[threadIdx.x >> 5];
  for (int64_t r = warp; r < M; r += nwarps) {
    const uint16_t* row = x + r * ld_x;
    auto each = [&](auto f) {
      for (int64_t g = lane; g < groups; g += 32) {
        f(ldg16(row + g * 16));
        f(ldg16(row + g * 16 + 8));
      }
    };
    float a = 0.0f, b = 0.0f;
    bool fast = false, certified = false;
    if (!exact_only) {
      if constexpr (kLN) {
        double s1 = 0.0, s2 = 0.0;
        each([&](const uint4& v) { normstats::sums8(v, s1, s2); });
        s1 = normstats::warp_sum(s1);
        s2 = normstats::warp_sum(s2);
        fast = normstats::ln_fast(s1, s2, K, rK, &a, &b);
        if (!fast && ln_row_mean_exact(row, K, s1, s2, rK, &a, &b)) certified = true;
      } else {
        double acc = 0.0;
        each([&](const uint4& v) { acc = normstats::sumsq8(v, acc); });
        acc = normstats::warp_sum(acc);
        fast = normstats::ms_fast(acc, K, rK, &a);
      }
    }
    if (!fast && !certified) norm_row_exact<kLN>(row, K, xs, &a, &b);
    if (lane == 0) {
      stat0[r] = a;
      if (stat1) stat1[r] = b;
      if (path) path[r] = fast ? 0 : (certified ? 2 : 1);
    }
  }
}

// ---------------------------------------------------------------------------
// MXFP8.
// ---------------------------------------------------------------------------
// Scale exponent e (and the multiplier 2^-e) of a group with |amax| bits `mag`.
__device__ __forceinline__ void mx_scale(uint32_t mag, uint32_t& sfb, float& mul) {
  int E;
  if (mag >= 0x80u)
    E = static_cast<int>(mag >> 7) - 127;                       // normal: exponent field
  else if (mag != 0u)
    E = (31 - __clz(static_cast<int>(mag))) - 133;              // subnormal: m * 2^-133
  else
    E = -100000;                                                // amax 0: log2 = -inf
  int e = E - 8;                                                // 8: exponent of 448, the e4m3 max
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  sfb = static_cast<uint32_t>(e + 127);
  mul = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e, exact (e <= 119 for finite bf16)
}

__device__ __forceinline__ uint2 mx_elems8(const uint4& v, float mul) {
  uint2 o;
  o.x = cvt_e4m3x2(__fmul_rn(bf16_bits_to_f32(v.x & 0xFFFFu), mul), __fmul_rn(bf16_bits_to_f32(v.x >> 16), mul)) |
        (cvt_e4m3x2(__fmul_rn(bf16_bits_to_f32(v.y & 0xFFFFu), mul), __fmul_rn(bf16_bits_to_f32(v.y >> 16), mul))
         << 16);
  o.y = cvt_e4m3x2(__fmul_rn(bf16_bits_to_f32(v.z & 0xFFFFu), mul), __fmul_rn(bf16_bits_to_f32(v.z >> 16), mul)) |
        (cvt_e4m3x2(__fmul_rn(bf16_bits_to_f32(v.w & 0xFFFFu), mul), __fmul_rn(bf16_bits_to_f32(v.w >> 16), mul))
         << 16);
  return o;
}

// K % 128 == 0: one lane quantizes one group of 32 (four adjacent 16-byte
// loads); a warp step covers 32 groups = 1024 elements of one row.
template <int U>
__device__ __forceinline__ void mxfp8_steps(const uint16_t* lp, uint8_t* qp, uint8_t* sp, bool live, bool store_sf) {
  uint4 v[U][4];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) v[u][i] = live ? ldg16(lp + u * 1024 + i * 8) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const uint32_t mag = max_of_halves<InBf16>(__hmax2(__hmax2(absmax8_x2<InBf16>(v[u][0]), absmax8_x2<InBf16>(v[u][1])),
                                                       __hmax2(absmax8_x2<InBf16>(v[u][2]), absmax8_x2<InBf16>(v[u][3]))));
    uint32_t sfb;
    float mul;
    mx_scale(mag, sfb, mul);
    const uint2 o0 = mx_elems8(v[u][0], mul), o1 = mx_elems8(v[u][1], mul);
    const uint2 o2 = mx_elems8(v[u][2], mul), o3 = mx_elems8(v[u][3], mul);
    const uint32_t s1 = __shfl_down_sync(kFull, sfb, 1);
    const uint32_t s2 = __shfl_down_sync(kFull, sfb, 2);
    const uint32_t s3 = __shfl_down_sync(kFull, sfb, 3);
    if (live) {
      *reinterpret_cast<uint4*>(qp + u * 1024) = make_uint4(o0.x, o0.y, o1.x, o1.y);
      *reinterpret_cast<uint4*>(qp + u * 1024 + 16) = make_uint4(o2.x, o2.y, o3.x, o3.y);
    }
    if (store_sf) *reinterpret_cast<uint32_t*>(sp + u * 4096) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
  }
}

__global__ void __launch_bounds__(kQuantThreads) mxfp8_quant_k128_kernel(const uint16_t* __restrict__ x, int64_t M,
                                                                          int64_t Mp, int64_t K, int64_t ld_x,
                                                                          uint8_t* __restrict__ q,
                                                                          uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  const uint32_t lane = lane_id();
  const int64_t groups = K >> 5;
  const int64_t steps = groups >> 5;
  const int64_t rem = groups & 31;  // a multiple of 4
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const bool quad_lead = (lane & 3u) == 0u;
  constexpr int kU = 2;

  for (int64_t r = warp; r < Mp; r += nwarps) {
    const bool live = r < M;
    const uint16_t* lp = x + r * ld_x + lane * 32;
    uint8_t* qp = q + r * K + lane * 32;
    uint8_t* sp = sf + Sf128x4::row_base(r, groups >> 2) + (lane >> 2) * 512;
    int64_t st = 0;
    for (; st + kU <= steps; st += kU) mxfp8_steps<kU>(lp + st * 1024, qp + st * 1024, sp + st * 4096, live, quad_lead);
    for (; st < steps; ++st) mxfp8_steps<1>(lp + st * 1024, qp + st * 1024, sp + st * 4096, live, quad_lead);
    if (rem) {
      const bool in = lane < rem;
      mxfp8_steps<1>(in ? lp + st * 1024 : lp, in ? qp + st * 1024 : qp, in ? sp + st * 4096 : sp, live && in,
                     in && quad_lead);
    }
  }
}

// Any K % 32 == 0: one warp per row, one lane per group of 32.
__global__ void __launch_bounds__(kQuantThreads) mxfp8_quant_generic_kernel(const uint16_t* __restrict__ x,
                                                                             int64_t M, int64_t Mp, int64_t K,
                                                                             int64_t ld_x, uint8_t* __restrict__ q,
                                                                             uint8_t* __restrict__ sf) {
  allow_dependent_launch();  // the GEMM that consumes this output may set up meanwhile
  const uint32_t lane = lane_id();
  const int64_t groups = K >> 5, cols4 = (groups + 3) & ~int64_t(3);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = warp; r < Mp; r += nwarps) {
    const bool live = r < M;
    const uint16_t* row = x + r * ld_x;
    const int64_t sfb_row = Sf128x4::row_base(r, cols4 >> 2);
    for (int64_t c = lane; c < cols4; c += 32) {
      uint32_t sfb = 0;
      if (live && c < groups) {
        uint4 v[4];
        uint32_t mag = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[i] = ldg16(row + c * 32 + i * 8);
          mag = max(mag, max_mag8<InBf16>(v[i]));
        }
        float mul;
        mx_scale(mag, sfb, mul);
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint2*>(q + r * K + c * 32 + i * 8) = mx_elems8(v[i], mul);
      }
      sf[sfb_row + (c >> 2) * 512 + (c & 3)] = static_cast<uint8_t>(sfb);
    }
  }
}

// ---------------------------------------------------------------------------
// Global scales.
// ---------------------------------------------------------------------------
template <class In>
__global__ void __launch_bounds__(kQuantThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                              uint32_t* __restrict__ amax_bits) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t nvec = n >> 3;
  uint32_t m = 0;
  for (int64_t i = tid; i < nvec; i += nthreads) m = max(m, max_sane_mag8<In>(ldg16(x + i * 8)));
  for (int64_t i = (nvec << 3) + tid; i < n; i += nthreads) m = max(m, sane_mag<In>(x[i]));
  m = warp_max(m);
  __shared__ uint32_t red[kQuantThreads / 32];
  if (lane_id() == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0u;
    m = warp_max(m);
    // a non-negative fp32 bit pattern: integer order == value order
    if (threadIdx.x == 0 && m != 0u) atomicMax(amax_bits, __float_as_uint(In::value(m)));
  }
}

__global__ void global_scale_kernel(const float* __restrict__ amax, float fp8_fp4_max, float* gs, float* inv_gs) {
  const float a = *amax;
  const float g = (a > 0.0f) ? __fdiv_rn(fp8_fp4_max, a) : 1.0f;
  if (gs) *gs = g;
  if (inv_gs) *inv_gs = __fdiv_rn(1.0f, g);
}

// ---------------------------------------------------------------------------
// Load-time weight conversion in one launch (the weight path of
// sgl-project sglang nvfp4_online.py, _quantize_weight_nvfp4, and of
// hao-ai-lab-FastVideo nvfp4_config.py: amax, then gs_w = fp8_fp4_max / amax,
// then the NVFP4 quantization with gs_w), K % 64 == 0:
//   1. every block folds its share of max|w| (sanitized as bsp_amax) into one
//      word of the workspace;
//   2. grid barrier;
//   3. every block reduces the words to amax and derives gs and 1/gs exactly as
//      bsp_nvfp4_global_scale_max; block 0 stores them;
//   4. the rows are quantized with gs by nvfp4_row_k64, last row first, so the
//      rows phase 1 read last are re-read from L2 rather than DRAM (a weight
//      smaller than L2 is read from DRAM once).
// The grid is one co-resident wave (a cooperative launch where the runtime
// allows it), so every block reaches the barrier.
// Workspace: [0] arrivals at the barrier, [1] barrier generation (both set to
// 0 on the stream before every launch), then one word per block from byte
// kWeightWsHeader.
// ---------------------------------------------------------------------------
constexpr int64_t kWeightWsHeader = 256;
constexpr int kWeightBatchMax = BSP_WEIGHT_BATCH_MAX;  // weights per nvfp4_quantize_weights call
#ifndef BSP_WQ_AMAX_LOADS
#define BSP_WQ_AMAX_LOADS 8  // 16-byte loads in flight per thread in the amax phase
#endif
#ifndef BSP_WQ_ROW_STEPS
#define BSP_WQ_ROW_STEPS 4  // warp steps in flight per row in the quantize phase
#endif
#ifndef BSP_WQ_MIN_BLOCKS
#define BSP_WQ_MIN_BLOCKS 1
#endif

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// All blocks of the grid meet here (bounded: false after kWaitLimitNs, with the
// error word raised).  The last block to arrive resets the arrival count and
// advances the generation, which releases the others.
__device__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t nblocks, uint32_t* err) {
  __shared__ int ok_sh;
  __syncthreads();
  if (threadIdx.x == 0) {
    bool ok = true;
    __threadfence();  // this block's writes are visible before its arrival
    const uint32_t g0 = ld_acquire_gpu(gen);
    if (atomicAdd(count, 1u) == nblocks - 1u) {
      atomicExch(count, 0u);
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_gpu(gen) == g0) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          ok = false;
          raise_error(err, kErrTimeout);
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    ok_sh = ok ? 1 : 0;
  }
  __syncthreads();
  return ok_sh != 0;
}

// Block-wide max of a per-thread magnitude, returned to every thread.
__device__ __forceinline__ uint32_t block_max(uint32_t m) {
  __shared__ uint32_t red[kQuantThreads / 32];
  m = warp_max(m);
  __syncthreads();  // red may still be read from a previous call
  if (lane_id() == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = lane_id() < kQuantThreads / 32 ? red[lane_id()] : 0u;
  return warp_max(m);
}

// Phase 1: this block's max|w| (sanitized magnitudes as in amax_kernel), the
// block's threads striding over the whole grid's share.
template <class In>
__device__ __forceinline__ uint32_t weight_block_amax(const uint16_t* __restrict__ w, int64_t N, int64_t K,
                                                      int64_t ld_w) {
  const uint32_t lane = lane_id();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  uint32_t m = 0;
  if (ld_w == K) {
    constexpr int A = BSP_WQ_AMAX_LOADS;
    const int64_t nvec = (N * K) >> 3;
    int64_t i = tid;
    for (; i + (A - 1) * nthreads < nvec; i += A * nthreads) {
      uint4 v[A];
#pragma unroll
      for (int j = 0; j < A; ++j) v[j] = ldg16(w + (i + j * nthreads) * 8);
#pragma unroll
      for (int j = 0; j < A; ++j) m = max(m, max_sane_mag8<In>(v[j]));
    }
    for (; i < nvec; i += nthreads) m = max(m, max_sane_mag8<In>(ldg16(w + i * 8)));
  } else {
    for (int64_t r = tid >> 5; r < N; r += nthreads >> 5)
      for (int64_t c = lane * 8; c < K; c += 256) m = max(m, max_sane_mag8<In>(ldg16(w + r * ld_w + c)));
  }
  return block_max(m);
}

// Phase 3: amax from the blocks' words (read through L2: other SMs wrote
// them) and gs exactly as bsp_nvfp4_global_scale_max; block 0 stores them.
template <class In>
__device__ __forceinline__ float weight_global_scale(const uint32_t* part, float fp8_fp4_max, float* amax_out,
                                                     float* gs_out, float* inv_out) {
  uint32_t m = 0;
  for (int64_t i = threadIdx.x; i < gridDim.x; i += blockDim.x) m = max(m, __ldcg(part + i));
  m = block_max(m);
  const float amax = m == 0u ? 0.0f : In::value(m);
  const float gs = amax > 0.0f ? __fdiv_rn(fp8_fp4_max, amax) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (amax_out) *amax_out = amax;
    if (gs_out) *gs_out = gs;
    if (inv_out) *inv_out = __fdiv_rn(1.0f, gs);
  }
  return gs;
}

// Phase 4: the rows, last row first, one warp per row.
template <class In>
__device__ __forceinline__ void weight_rows(const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ld_w,
                                            float gs, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int64_t Np = (N + 127) / 128 * 128;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < Np; i += nwarps) {
    const int64_t r = Np - 1 - i;
    const bool live = r < N;
    nvfp4_row_k64<In, Sf128x4, BSP_WQ_ROW_STEPS>(w + (live ? r : 0) * ld_w, K, r, live, gs, codes, sf, lane_id(),
                                                 nullptr);
  }
}

template <class In>
__global__ void __launch_bounds__(kQuantThreads, BSP_WQ_MIN_BLOCKS) nvfp4_weight_kernel(
    const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ld_w, float fp8_fp4_max,
    float* __restrict__ amax_out, float* __restrict__ gs_out, float* __restrict__ inv_out, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf, uint8_t* __restrict__ ws, uint32_t* __restrict__ err) {
  uint32_t* count = reinterpret_cast<uint32_t*>(ws);
  uint32_t* part = reinterpret_cast<uint32_t*>(ws + kWeightWsHeader);
  const uint32_t m = weight_block_amax<In>(w, N, K, ld_w);                      // 1.
  if (threadIdx.x == 0) part[blockIdx.x] = m;
  if (!grid_barrier(count, count + 1, gridDim.x, err)) return;                  // 2.
  const float gs = weight_global_scale<In>(part, fp8_fp4_max, amax_out, gs_out, inv_out);  // 3.
  weight_rows<In>(w, N, K, ld_w, gs, codes, sf);                                 // 4.
}

// Many weights in one launch: the phases of nvfp4_weight_kernel per weight,
// one grid barrier each.  A block that has quantized its rows of weight j goes
// on to the amax of weight j + 1 while others finish, so one weight's tail
// overlaps the next one's reads.  The blocks' words alternate between two
// slots: slot j % 2 is rewritten (for weight j + 2) only after the barrier of
// weight j + 1, which every block passes after reading it.
struct WeightBatch {
  int count;
  bsp_weight_desc d[kWeightBatchMax];
};

template <class In>
__global__ void __launch_bounds__(kQuantThreads, 3) nvfp4_weights_kernel(
    const __grid_constant__ WeightBatch batch, float fp8_fp4_max, uint8_t* __restrict__ ws, uint32_t* __restrict__ err) {
  uint32_t* count = reinterpret_cast<uint32_t*>(ws);
  uint32_t* part = reinterpret_cast<uint32_t*>(ws + kWeightWsHeader);
  for (int j = 0; j < batch.count; ++j) {
    const bsp_weight_desc& d = batch.d[j];
    uint32_t* slot = part + (j & 1) * gridDim.x;
    const uint32_t m = weight_block_amax<In>(d.w, d.N, d.K, d.ld_w);
    if (threadIdx.x == 0) slot[blockIdx.x] = m;
    if (!grid_barrier(count, count + 1, gridDim.x, err)) return;
    const float gs = weight_global_scale<In>(slot, fp8_fp4_max, d.amax, d.gs, d.inv_gs);
    weight_rows<In>(d.w, d.N, d.K, d.ld_w, gs, d.codes, d.sf);
  }
}

__global__ void alpha_kernel(const float* __restrict__ gs_x, const float* __restrict__ gs_w, float* alpha) {
  *alpha = __fdiv_rn(1.0f, __fmul_rn(*gs_x, *gs_w));
}

// ---------------------------------------------------------------------------
// Diagnostics.
// ---------------------------------------------------------------------------
__global__ void debug_e2m1_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = static_cast<uint8_t>(cvt_e2m1x8(v[i], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 0xFu);
}

__global__ void debug_e4m3_kernel(const float* __restrict__ v, int64_t n, uint8_t* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = static_cast<uint8_t>(cvt_e4m3x2(v[i], 0.f) & 0xFFu);
}

__global__ void debug_wait_kernel(uint64_t limit_ns, uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, nullptr, limit_ns)) raise_error(err, kErrTimeout);
}

// Persistent grid: exactly the blocks that are resident at once (rows are
// spread over warps by a grid-stride loop), so no block starts in a second,
// partial wave.
template <typename Kernel>
int grid_for_rows(const DeviceInfo& dev, Kernel kernel, int64_t rows, size_t dynamic_smem = 0) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQuantThreads, dynamic_smem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const int64_t warps_per_block = kQuantThreads / 32;
  const int64_t needed = ceil_div(rows, warps_per_block);
  const int64_t cap = static_cast<int64_t>(dev.sm_count) * per_sm;
  return static_cast<int>(needed < cap ? (needed > 0 ? needed : 1) : cap);
}

// max|x| folded into *amax (zeroed first when `reset`).
template <class In>
int amax_launch(const uint16_t* x, int64_t n, float* amax, cudaStream_t stream, bool reset) {
  if (n < 0 || !amax || (n > 0 && !x)) return BSP_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || (reinterpret_cast<uintptr_t>(amax) & 3u)) return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (reset && cudaMemsetAsync(amax, 0, sizeof(float), stream) != cudaSuccess) return launch_status();
  if (n == 0) return BSP_OK;
  int64_t blocks = ceil_div(ceil_div(n, 8), kQuantThreads);
  const int64_t cap = static_cast<int64_t>(dev.sm_count) * 8;
  if (blocks > cap) blocks = cap;
  amax_kernel<In><<<static_cast<int>(blocks), kQuantThreads, 0, stream>>>(x, n, reinterpret_cast<uint32_t*>(amax));
  return launch_status();
}

// Per-token quantize of a row that fits registers (K = 1024, 1536, 2048 or
// 5120).  Warps per row S: enough that each SM gets about kRowWarpsPerSm of
// them -- the fewest for many rows, up to one group a thread for a handful of
// rows; teams per block fill 8 warps where rows allow.
constexpr int kRowWarpsPerSm = 16;

template <class In, class L>
int launch_rowreg(const DeviceInfo& dev, const uint16_t* x, int64_t M, int64_t Mp, int64_t K, int64_t ld_x,
                  float* row_gs, float* row_inv, uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  const int gk = static_cast<int>(K / 512);  // S * G
  // warps per live row wanted (padding rows [M, Mp) load nothing); at most 5
  // groups a thread (K = 5120 on one warp holds 120 registers a thread, and its
  // low occupancy measured slower than two warps a row at every row count)
  const int64_t want = ceil_div(static_cast<int64_t>(dev.sm_count) * kRowWarpsPerSm, M);
  int S = 0;
  for (int s = 1; s <= gk && s <= 8; ++s)
    if (gk % s == 0 && gk / s <= 5 && (S == 0 || s <= want)) S = s;
  auto go = [&](auto k, int s) -> int {
    const int64_t teams_wanted = ceil_div(Mp, static_cast<int64_t>(dev.sm_count));
    const int teams = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(teams_wanted, std::min(8 / s, kRowTeamMax))));
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, 32 * s * teams, 0) != cudaSuccess || per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    const int64_t blocks = std::min<int64_t>(ceil_div(Mp, teams), static_cast<int64_t>(dev.sm_count) * per_sm);
    k<<<static_cast<int>(blocks), 32 * s * teams, 0, stream>>>(x, M, Mp, ld_x, row_gs, row_inv, codes, sf);
    return BSP_OK;
  };
  switch (gk * 16 + S) {
    case 2 * 16 + 1: return go(nvfp4_quant_rowreg_kernel<In, L, 2, 1>, 1);
    case 2 * 16 + 2: return go(nvfp4_quant_rowreg_kernel<In, L, 1, 2>, 2);
    case 3 * 16 + 1: return go(nvfp4_quant_rowreg_kernel<In, L, 3, 1>, 1);
    case 3 * 16 + 3: return go(nvfp4_quant_rowreg_kernel<In, L, 1, 3>, 3);
    case 4 * 16 + 1: return go(nvfp4_quant_rowreg_kernel<In, L, 4, 1>, 1);
    case 4 * 16 + 2: return go(nvfp4_quant_rowreg_kernel<In, L, 2, 2>, 2);
    case 4 * 16 + 4: return go(nvfp4_quant_rowreg_kernel<In, L, 1, 4>, 4);
    case 10 * 16 + 2: return go(nvfp4_quant_rowreg_kernel<In, L, 5, 2>, 2);
    case 10 * 16 + 5: return go(nvfp4_quant_rowreg_kernel<In, L, 2, 5>, 5);
    default: return BSP_ERR_INVALID_ARG;
  }
}

template <class In, class L>
int run_nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* global_sf, int sf_mode,
                       float* row_gs, float* row_inv_gs, uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 16 != 0 || ld_x < K) return BSP_ERR_INVALID_ARG;
  if (sf_mode != BSP_SF_PER_TENSOR && sf_mode != BSP_SF_PER_ROW) return BSP_ERR_INVALID_ARG;
  if (M == 0) return BSP_OK;
  if (!x || !codes || !sf || (sf_mode == BSP_SF_PER_TENSOR && !global_sf)) return BSP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ld_x % 8 != 0) return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  const int64_t Mp = round_up(M, L::kRowTile);
  const bool per_row = sf_mode == BSP_SF_PER_ROW;
  if (K % 64 == 0) {
    int rowblock_cap = 0;  // rows the block-per-row kernel keeps resident at once
    if (per_row && K <= 16 * kQuantThreads * kRowG) {
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, nvfp4_quant_rowblock_kernel<In, L>, kQuantThreads,
                                                        0) != cudaSuccess ||
          per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
      }
      rowblock_cap = dev.sm_count * per_sm;
    }
    if (per_row && (K == 1024 || K == 1536 || K == 2048 || K == 5120)) {
      st = launch_rowreg<In, L>(dev, x, M, Mp, K, ld_x, row_gs, row_inv_gs, codes, sf, stream);
      if (st != BSP_OK) return st;
    } else if (per_row && Mp <= rowblock_cap) {
      // few rows: one block per row, all rows in one wave, one memory round trip
      nvfp4_quant_rowblock_kernel<In, L><<<static_cast<int>(Mp), kQuantThreads, 0, stream>>>(x, M, Mp, K, ld_x, row_gs,
                                                                                      row_inv_gs, codes, sf);
    } else if (per_row) {
      auto k = nvfp4_quant_k64_kernel<In, L, true>;
      k<<<grid_for_rows(dev, k, Mp), kQuantThreads, 0, stream>>>(x, M, Mp, K, ld_x, global_sf, row_gs, row_inv_gs,
                                                                 codes, sf);
    } else if (K == 1024 || K == 1536) {
      const int64_t pairs = ceil_div(Mp, 2);
      if (K == 1024) {
        auto k = nvfp4_quant_short_kernel<In, L, 2>;
        k<<<grid_for_rows(dev, k, pairs), kQuantThreads, 0, stream>>>(x, M, Mp, ld_x, global_sf, codes, sf);
      } else {
        auto k = nvfp4_quant_short_kernel<In, L, 3>;
        k<<<grid_for_rows(dev, k, pairs), kQuantThreads, 0, stream>>>(x, M, Mp, ld_x, global_sf, codes, sf);
      }
    } else {
      auto k = nvfp4_quant_k64_kernel<In, L, false>;
      k<<<grid_for_rows(dev, k, Mp), kQuantThreads, 0, stream>>>(x, M, Mp, K, ld_x, global_sf, nullptr, nullptr,
                                                                 codes, sf);
    }
  } else {
    if (per_row) {
      auto k = nvfp4_quant_generic_kernel<In, L, true>;
      k<<<grid_for_rows(dev, k, Mp), kQuantThreads, 0, stream>>>(x, M, Mp, K, ld_x, global_sf, row_gs, row_inv_gs,
                                                                 codes, sf);
    } else {
      auto k = nvfp4_quant_generic_kernel<In, L, false>;
      k<<<grid_for_rows(dev, k, Mp), kQuantThreads, 0, stream>>>(x, M, Mp, K, ld_x, global_sf, nullptr, nullptr,
                                                                 codes, sf);
    }
  }
  return launch_status();
}

// Blocks of nvfp4_weight_kernel<In> resident at once on this device: its grid.
template <class In>
int weight_grid(const DeviceInfo& dev, int* grid) {
  int per_sm = 0;
  int per_sm_batch = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, nvfp4_weight_kernel<In>, kQuantThreads, 0) !=
          cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_batch, nvfp4_weights_kernel<In>, kQuantThreads, 0) !=
          cudaSuccess ||
      per_sm < 1 || per_sm_batch < 1)
    return (cudaGetLastError(), BSP_ERR_CUDA);
  // one grid for both kernels (they share the workspace layout): the smaller residency
  *grid = dev.sm_count * (per_sm < per_sm_batch ? per_sm : per_sm_batch);
  return BSP_OK;
}

template <class In>
int run_nvfp4_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int64_t ld_w, float fp8_fp4_max, float* amax,
                              float* gs, float* inv_gs, uint8_t* codes, uint8_t* sf, void* ws, int64_t ws_bytes,
                              cudaStream_t stream) {
  if (N < 0 || K <= 0 || K % 64 != 0 || ld_w < K) return BSP_ERR_INVALID_ARG;
  if (!(fp8_fp4_max > 0.0f) || !(fp8_fp4_max <= 3.4028234663852886e38f)) return BSP_ERR_INVALID_ARG;
  if ((N > 0 && !w) || !codes || !sf || !gs || !inv_gs || !ws) return BSP_ERR_INVALID_ARG;
  if ((w && !aligned16(w)) || !aligned16(codes) || !aligned16(sf) || !aligned16(ws) || ld_w % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(gs) & 3u) || (reinterpret_cast<uintptr_t>(inv_gs) & 3u) ||
      (reinterpret_cast<uintptr_t>(amax) & 3u))
    return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  int grid = 0;
  if ((st = weight_grid<In>(dev, &grid)) != BSP_OK) return st;
  if (ws_bytes < kWeightWsHeader + 4 * static_cast<int64_t>(grid)) return BSP_ERR_INVALID_ARG;  // one slot used here
  // the barrier words start at 0 whatever an earlier call left (one that timed
  // out leaves its arrival count behind)
  if (cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), stream) != cudaSuccess) return launch_status();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeCooperative;  // all blocks resident at once, or no launch
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, nvfp4_weight_kernel<In>, w, N, K, ld_w, fp8_fp4_max, amax, gs, inv_gs, codes, sf,
                         static_cast<uint8_t*>(ws), dev.err_word) != cudaSuccess)
    return launch_status();
  return BSP_OK;
}

template <class In>
int run_nvfp4_quantize_weights(const bsp_weight_desc* descs, int count, float fp8_fp4_max, void* ws, int64_t ws_bytes,
                               cudaStream_t stream) {
  if (count < 0 || count > kWeightBatchMax || (count > 0 && !descs) || !ws) return BSP_ERR_INVALID_ARG;
  if (!(fp8_fp4_max > 0.0f) || !(fp8_fp4_max <= 3.4028234663852886e38f)) return BSP_ERR_INVALID_ARG;
  WeightBatch batch;
  batch.count = count;
  for (int j = 0; j < count; ++j) {
    const bsp_weight_desc& d = descs[j];
    if (d.N < 0 || d.K <= 0 || d.K % 64 != 0 || d.ld_w < d.K) return BSP_ERR_INVALID_ARG;
    if ((d.N > 0 && !d.w) || !d.codes || !d.sf || !d.gs || !d.inv_gs) return BSP_ERR_INVALID_ARG;
    if ((d.w && !aligned16(d.w)) || !aligned16(d.codes) || !aligned16(d.sf) || d.ld_w % 8 != 0 ||
        (reinterpret_cast<uintptr_t>(d.gs) & 3u) || (reinterpret_cast<uintptr_t>(d.inv_gs) & 3u) ||
        (reinterpret_cast<uintptr_t>(d.amax) & 3u))
      return BSP_ERR_ALIGNMENT;
    batch.d[j] = d;
  }
  if (!aligned16(ws)) return BSP_ERR_ALIGNMENT;
  if (count == 0) return BSP_OK;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  int grid = 0;
  if ((st = weight_grid<In>(dev, &grid)) != BSP_OK) return st;
  if (ws_bytes < kWeightWsHeader + 8 * static_cast<int64_t>(grid)) return BSP_ERR_INVALID_ARG;
  if (cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), stream) != cudaSuccess) return launch_status();  // barrier words
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeCooperative;  // all blocks resident at once, or no launch
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, nvfp4_weights_kernel<In>, batch, fp8_fp4_max, static_cast<uint8_t*>(ws),
                         dev.err_word) != cudaSuccess)
    return launch_status();
  return BSP_OK;
}

// Scratch of nvfp4_quantize_weight_static: a file-scope device array (no
// allocation by anyone) that holds the reported workspace size (header and two
// words per block) for grids of up to kStaticWeightWsBlocks / 2 blocks.
constexpr int64_t kStaticWeightWsBlocks = 4096;
constexpr int64_t kStaticWeightWsBytes = kWeightWsHeader + 4 * kStaticWeightWsBlocks;
static __device__ __align__(256) uint8_t g_weight_ws[kStaticWeightWsBytes];

// Its address on device dev.id, looked up once per device (the launch clears
// the barrier words before every call).  The set-up is serialised by a lock;
// the first call must come before any stream capture (the symbol lookup may
// load the module).  The cached address belongs to the device's primary
// context: after cudaDeviceReset the entry is not to be called again in the
// same process.
int static_weight_ws(const DeviceInfo& dev, void** out) {
  static void* addr[64] = {};
  static std::mutex mu;
  if (dev.id < 0 || dev.id >= 64) return BSP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev.id]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_weight_ws) != cudaSuccess) return launch_status();
    addr[dev.id] = p;
  }
  *out = addr[dev.id];
  return BSP_OK;
}

// Largest K of the fused norms: the exact path's digit counts and its 32-bit
// divisor (K for the mean of squares, K^2 for the variance) bound it.
constexpr int64_t norm_max_k(bool ln) { return ln ? 32768 : (int64_t(1) << 20); }

template <bool kLN>
int run_norm_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const uint16_t* gamma,
                      const uint16_t* beta, float eps, const float* global_sf, int sf_mode, float* row_gs,
                      float* row_inv_gs, float* row_mean, float* row_rstd, uint8_t* codes, uint8_t* sf,
                      cudaStream_t stream) {
  if (M < 0 || K <= 0 || K % 16 != 0 || ld_x < K || K > norm_max_k(kLN)) return BSP_ERR_INVALID_ARG;
  if (sf_mode != BSP_SF_PER_TENSOR && sf_mode != BSP_SF_PER_ROW) return BSP_ERR_INVALID_ARG;
  if (!(eps >= 0.0f) || !(eps <= 3.4028234663852886e38f)) return BSP_ERR_INVALID_ARG;
  if (M == 0) return BSP_OK;
  if (!x || !codes || !sf || (sf_mode == BSP_SF_PER_TENSOR && !global_sf)) return BSP_ERR_INVALID_ARG;
  if (!aligned16(x) || (gamma && !aligned16(gamma)) || (beta && !aligned16(beta)) || !aligned16(codes) ||
      !aligned16(sf) || ld_x % 8 != 0)
    return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  const int64_t Mp = round_up(M, 128);
  const bool per_row = sf_mode == BSP_SF_PER_ROW;
  float* rg = per_row ? row_gs : nullptr;
  float* ri = per_row ? row_inv_gs : nullptr;
  // K = 1536 / 2048: rows in registers (at K = 1024 the multi-pass kernel
  // below measured as fast)
  if (K == 1536 || K == 2048) {
    auto launch = [&](auto k, int64_t rows_per_warp) {
      k<<<grid_for_rows(dev, k, ceil_div(Mp, rows_per_warp)), kQuantThreads, 0, stream>>>(
          x, M, Mp, ld_x, gamma, beta, eps, global_sf, rg, ri, row_mean, row_rstd, codes, sf);
    };
    switch (K / 512) {
#define BSP_NORM_CASE(S_, R_, B_)                                                                      \
  case S_:                                                                                            \
    per_row ? launch(nvfp4_norm_quant_short_kernel<true, kLN, S_, R_, B_>, R_)                        \
            : launch(nvfp4_norm_quant_short_kernel<false, kLN, S_, R_, B_>, R_);                      \
    break;
      BSP_NORM_CASE(3, BSP_RMSNORM_ROWS, BSP_RMSNORM_MIN_BLOCKS)
      BSP_NORM_CASE(4, 1, 2)
#undef BSP_NORM_CASE
    }
    return launch_status();
  }
  const size_t stage = norm_stage_bytes(K, kLN);
  auto launch = [&](auto k, size_t smem) -> int {
    k<<<grid_for_rows(dev, k, Mp, smem), kQuantThreads, smem, stream>>>(x, M, Mp, K, ld_x, gamma, beta, eps, global_sf,
                                                                      rg, ri, row_mean, row_rstd, codes, sf);
    return launch_status();
  };
  if (stage <= kNormStageMaxBytes)
    return per_row ? launch(nvfp4_norm_quant_kernel<Sf128x4, true, kLN, true>, stage)
                   : launch(nvfp4_norm_quant_kernel<Sf128x4, false, kLN, true>, stage);
  return per_row ? launch(nvfp4_norm_quant_kernel<Sf128x4, true, kLN, false>, 0)
                 : launch(nvfp4_norm_quant_kernel<Sf128x4, false, kLN, false>, 0);
}

}  // namespace
}  // namespace bsp

using namespace bsp;

extern "C" {

int nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* global_sf, int sf_mode,
                   float* row_gs, float* row_inv_gs, uint8_t* codes, uint8_t* sf, bsp_stream_t stream) {
  return run_nvfp4_quantize<InBf16, Sf128x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf, stream);
}

int nvfp4_quantize_f16(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* global_sf, int sf_mode,
                       float* row_gs, float* row_inv_gs, uint8_t* codes, uint8_t* sf, bsp_stream_t stream) {
  return run_nvfp4_quantize<InF16, Sf128x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf, stream);
}

int nvfp4_quantize_ex(const uint16_t* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x, const float* global_sf,
                      int sf_mode, int sf_layout, float* row_gs, float* row_inv_gs, uint8_t* codes, uint8_t* sf,
                      bsp_stream_t stream) {
  if (x_dtype != BSP_IN_BF16 && x_dtype != BSP_IN_F16) return BSP_ERR_INVALID_ARG;
  if (sf_layout != BSP_SF_LAYOUT_128X4 && sf_layout != BSP_SF_LAYOUT_8X4) return BSP_ERR_INVALID_ARG;
  const bool f16 = x_dtype == BSP_IN_F16;
  if (sf_layout == BSP_SF_LAYOUT_8X4)
    return f16 ? run_nvfp4_quantize<InF16, Sf8x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf,
                                                  stream)
               : run_nvfp4_quantize<InBf16, Sf8x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf,
                                                   stream);
  return f16 ? run_nvfp4_quantize<InF16, Sf128x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf,
                                                  stream)
             : run_nvfp4_quantize<InBf16, Sf128x4>(x, M, K, ld_x, global_sf, sf_mode, row_gs, row_inv_gs, codes, sf,
                                                   stream);
}

int nvfp4_rmsnorm_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const uint16_t* gamma, float eps,
                           const float* global_sf, int sf_mode, float* row_gs, float* row_inv_gs, float* row_rstd,
                           uint8_t* codes, uint8_t* sf, bsp_stream_t stream) {
  if (!gamma && M > 0) return BSP_ERR_INVALID_ARG;
  return run_norm_quantize<false>(x, M, K, ld_x, gamma, nullptr, eps, global_sf, sf_mode, row_gs, row_inv_gs, nullptr,
                                  row_rstd, codes, sf, stream);
}

int nvfp4_layernorm_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const uint16_t* gamma,
                             const uint16_t* beta, float eps, const float* global_sf, int sf_mode, float* row_gs,
                             float* row_inv_gs, float* row_mean, float* row_rstd, uint8_t* codes, uint8_t* sf,
                             bsp_stream_t stream) {
  return run_norm_quantize<true>(x, M, K, ld_x, gamma, beta, eps, global_sf, sf_mode, row_gs, row_inv_gs, row_mean,
                                 row_rstd, codes, sf, stream);
}

int bsp_debug_norm_stats(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, int norm, int exact_only, float* stat0,
                         float* stat1, int* path, bsp_stream_t stream) {
  if (norm != BSP_NORM_RMS && norm != BSP_NORM_LAYER) return BSP_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 16 != 0 || ld_x < K || K > norm_max_k(norm == BSP_NORM_LAYER)) return BSP_ERR_INVALID_ARG;
  if (M == 0) return BSP_OK;
  if (!x || !stat0 || (norm == BSP_NORM_LAYER && !stat1)) return BSP_ERR_INVALID_ARG;
  if (!aligned16(x) || ld_x % 8 != 0) return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (norm == BSP_NORM_LAYER) {
    auto k = norm_stats_kernel<true>;
    k<<<grid_for_rows(dev, k, M), kQuantThreads, 0, stream>>>(x, M, K, ld_x, exact_only != 0, stat0, stat1, path);
  } else {
    auto k = norm_stats_kernel<false>;
    k<<<grid_for_rows(dev, k, M), kQuantThreads, 0, stream>>>(x, M, K, ld_x, exact_only != 0, stat0, nullptr, path);
  }
  return launch_status();
}

int mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, uint8_t* q, uint8_t* sf,
                   bsp_stream_t stream) {
  if (M < 0 || K <= 0 || K % 32 != 0 || ld_x < K) return BSP_ERR_INVALID_ARG;
  if (M == 0) return BSP_OK;
  if (!x || !q || !sf) return BSP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q) || !aligned16(sf) || ld_x % 8 != 0) return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  const int64_t Mp = round_up(M, 128);
  if (K % 128 == 0)
    mxfp8_quant_k128_kernel<<<grid_for_rows(dev, mxfp8_quant_k128_kernel, Mp), kQuantThreads, 0, stream>>>(
        x, M, Mp, K, ld_x, q, sf);
  else
    mxfp8_quant_generic_kernel<<<grid_for_rows(dev, mxfp8_quant_generic_kernel, Mp), kQuantThreads, 0, stream>>>(
        x, M, Mp, K, ld_x, q, sf);
  return launch_status();
}

int bsp_amax_bf16(const uint16_t* x, int64_t n, float* amax, bsp_stream_t stream) {
  return amax_launch<InBf16>(x, n, amax, stream, true);
}

int bsp_amax_bf16_into(const uint16_t* x, int64_t n, float* amax, bsp_stream_t stream) {
  return amax_launch<InBf16>(x, n, amax, stream, false);
}

int bsp_amax_f16(const uint16_t* x, int64_t n, float* amax, bsp_stream_t stream) {
  return amax_launch<InF16>(x, n, amax, stream, true);
}

int bsp_amax_f16_into(const uint16_t* x, int64_t n, float* amax, bsp_stream_t stream) {
  return amax_launch<InF16>(x, n, amax, stream, false);
}

int bsp_nvfp4_global_scale_max(const float* amax, float fp8_fp4_max, float* gs, float* inv_gs,
                               bsp_stream_t stream) {
  if (!amax || (!gs && !inv_gs)) return BSP_ERR_INVALID_ARG;
  if (!(fp8_fp4_max > 0.0f) || !(fp8_fp4_max <= 3.4028234663852886e38f)) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  global_scale_kernel<<<1, 1, 0, stream>>>(amax, fp8_fp4_max, gs, inv_gs);
  return launch_status();
}

int bsp_nvfp4_quantize_weight_workspace_bytes(int w_dtype, int64_t* bytes) {
  if (!bytes || (w_dtype != BSP_IN_BF16 && w_dtype != BSP_IN_F16)) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  int grid = 0;
  st = w_dtype == BSP_IN_F16 ? weight_grid<InF16>(dev, &grid) : weight_grid<InBf16>(dev, &grid);
  if (st != BSP_OK) return st;
  *bytes = kWeightWsHeader + 8 * static_cast<int64_t>(grid);  // two slots: enough for nvfp4_quantize_weights too
  return BSP_OK;
}

int nvfp4_quantize_weight(const uint16_t* w, int w_dtype, int64_t N, int64_t K, int64_t ld_w, float fp8_fp4_max,
                          float* amax, float* gs, float* inv_gs, uint8_t* codes, uint8_t* sf, void* workspace,
                          int64_t workspace_bytes, bsp_stream_t stream) {
  if (w_dtype == BSP_IN_F16)
    return run_nvfp4_quantize_weight<InF16>(w, N, K, ld_w, fp8_fp4_max, amax, gs, inv_gs, codes, sf, workspace,
                                            workspace_bytes, stream);
  if (w_dtype != BSP_IN_BF16) return BSP_ERR_INVALID_ARG;
  return run_nvfp4_quantize_weight<InBf16>(w, N, K, ld_w, fp8_fp4_max, amax, gs, inv_gs, codes, sf, workspace,
                                           workspace_bytes, stream);
}

int nvfp4_quantize_weight_static(const uint16_t* w, int w_dtype, int64_t N, int64_t K, int64_t ld_w,
                                 float fp8_fp4_max, float* amax, float* gs, float* inv_gs, uint8_t* codes, uint8_t* sf,
                                 bsp_stream_t stream) {
  if (w_dtype != BSP_IN_BF16 && w_dtype != BSP_IN_F16) return BSP_ERR_INVALID_ARG;
  // the host checks of nvfp4_quantize_weight, before the set-up touches the device
  if (N < 0 || K <= 0 || K % 64 != 0 || ld_w < K) return BSP_ERR_INVALID_ARG;
  if (!(fp8_fp4_max > 0.0f) || !(fp8_fp4_max <= 3.4028234663852886e38f)) return BSP_ERR_INVALID_ARG;
  if ((N > 0 && !w) || !codes || !sf || !gs || !inv_gs) return BSP_ERR_INVALID_ARG;
  int64_t need = 0;
  int st = bsp_nvfp4_quantize_weight_workspace_bytes(w_dtype, &need);
  if (st != BSP_OK) return st;
  if (need > kStaticWeightWsBytes) return BSP_ERR_INVALID_ARG;  // grid larger than the static scratch holds
  DeviceInfo dev;
  if ((st = current_device(&dev)) != BSP_OK) return st;
  void* ws = nullptr;
  if ((st = static_weight_ws(dev, &ws)) != BSP_OK) return st;
  return nvfp4_quantize_weight(w, w_dtype, N, K, ld_w, fp8_fp4_max, amax, gs, inv_gs, codes, sf, ws,
                               kStaticWeightWsBytes, stream);
}

int nvfp4_quantize_weights(const bsp_weight_desc* descs, int count, int w_dtype, float fp8_fp4_max, void* workspace,
                           int64_t workspace_bytes, bsp_stream_t stream) {
  if (w_dtype == BSP_IN_F16)
    return run_nvfp4_quantize_weights<InF16>(descs, count, fp8_fp4_max, workspace, workspace_bytes, stream);
  if (w_dtype != BSP_IN_BF16) return BSP_ERR_INVALID_ARG;
  return run_nvfp4_quantize_weights<InBf16>(descs, count, fp8_fp4_max, workspace, workspace_bytes, stream);
}

int bsp_nvfp4_global_scale(const float* amax, float* gs, float* inv_gs, bsp_stream_t stream) {
  return bsp_nvfp4_global_scale_max(amax, 448.0f * 6.0f, gs, inv_gs, stream);
}

int bsp_nvfp4_alpha(const float* gs_x, const float* gs_w, float* alpha, bsp_stream_t stream) {
  if (!gs_x || !gs_w || !alpha) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  alpha_kernel<<<1, 1, 0, stream>>>(gs_x, gs_w, alpha);
  return launch_status();
}

int bsp_debug_encode_e2m1(const float* v, int64_t n, uint8_t* codes, bsp_stream_t stream) {
  if (n < 0 || (n > 0 && (!v || !codes))) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (n == 0) return BSP_OK;
  debug_e2m1_kernel<<<static_cast<int>(ceil_div(n, 256)), 256, 0, stream>>>(v, n, codes);
  return launch_status();
}

int bsp_debug_encode_e4m3(const float* v, int64_t n, uint8_t* bytes, bsp_stream_t stream) {
  if (n < 0 || (n > 0 && (!v || !bytes))) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (n == 0) return BSP_OK;
  debug_e4m3_kernel<<<static_cast<int>(ceil_div(n, 256)), 256, 0, stream>>>(v, n, bytes);
  return launch_status();
}

int bsp_debug_wait_timeout(int64_t limit_ns, bsp_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000ll) return BSP_ERR_INVALID_ARG;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  debug_wait_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_ns), dev.err_word);
  return launch_status();
}

}  // extern "C"
