// gemm.cu -- block-scaled GEMM on sm_100a tensor cores (tcgen05):
//
//   D[m, n] = alpha * row_scale[m] * sum_k A(m,k) sA(m,k/g) B(n,k) sB(n,k/g) + bias[n]
//
// NVFP4: e2m1 operands, e4m3 scales per 16 (kind::mxf4nvf4, scale_vec::4X) --
//   hao-ai-lab-FastVideo nvfp4_qat_config.py, NVFP4QATQuantizeMethod.apply
//   (mm_fp4 of the packed activation and weight, alpha = 1/(gs_x*gs_w), bias
//   added after); nvfp4_config.py, _mm_fp4.
// MXFP8: e4m3 operands, e8m0 scales per 32 (kind::mxf8f6f4, scale_vec::1X) --
//   vllm-omni mxfp8_config.py, NPUMxfp8LinearMethod._quant_matmul.
//
// Design (one CTA per SM, persistent over output tiles of 128 x 256):
//   warp 0      TMA producer: per stage, 128 rows of A and 256 rows of B (128
//               bytes of K each, 128-byte swizzle) and the matching 128x4
//               scale tiles, all into shared memory, completion on an mbarrier.
//   warp 1      MMA issuer (one thread): copies the stage's scale tiles from
//               shared memory into tensor memory (tcgen05.cp), issues four
//               block-scaled MMAs (K = 64 fp4 / 32 fp8 each) accumulating into
//               a 128 x 256 fp32 accumulator in tensor memory, and releases the
//               stage with tcgen05.commit.
//   warps 2..9  epilogue, two warps per 32-lane quarter of tensor memory, each
//               owning 128 accumulator columns: read them into registers
//               (tcgen05.ld), hand the accumulator back to the MMA warp at once
//               (so the next tile's MMAs overlap this tile's stores), apply
//               alpha, row scale and bias in fp32, round once, stage 32 rows x
//               32 bytes in swizzled shared memory and write them with TMA
//               stores (full 32-byte sectors; rows/columns past M/N clipped).
// Tensor memory: columns [0, 256) accumulator; then, per pipeline stage, the
// stage's scale factors (a scale column may only be rewritten once the stage's
// MMAs have completed, which the stage's empty barrier already guarantees).
// Ragged M / N / K edges: TMA fills out-of-range rows, K bytes and scale tiles
// with zeros (zero codes times zero scales add nothing); TMA stores clip.
// Every wait is bounded; a wait that runs out raises the device error word and
// the CTA drains its outstanding copies and MMAs, frees tensor memory and exits.
#include "bsp_device.cuh"
#include "bsp_internal.h"

namespace bsp {
namespace {

enum Kind : int { kNVF4 = 0, kMXF8 = 1 };

template <int KIND>
struct Cfg {
  static constexpr int BM = 128, BN = 256;
  static constexpr int ROW_BYTES = 128;                 // K bytes per operand row per stage
  static constexpr int MMAS = 4;                         // per stage, 32 bytes of K each
  static constexpr int ATOMS = KIND == kNVF4 ? 4 : 1;    // 128x4 scale tiles per 128 rows per stage
  static constexpr int A_BYTES = BM * ROW_BYTES;
  static constexpr int B_BYTES = BN * ROW_BYTES;
  static constexpr int SFA_BYTES = ATOMS * 512;
  static constexpr int SFB_BYTES = 2 * ATOMS * 512;
  static constexpr int TX_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGE_BYTES = (TX_BYTES + 1023) / 1024 * 1024;
  static constexpr int STAGES = 4;
  static constexpr int SFA_COLS = ATOMS * 4;
  static constexpr int SFB_COLS = ATOMS * 8;
  static constexpr int SF_COLS = SFA_COLS + SFB_COLS;
  static constexpr int ACC_COLS = BN;
  static constexpr int TMEM_COLS = 512;
  static_assert(ACC_COLS + STAGES * SF_COLS <= TMEM_COLS, "tensor memory budget");
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_COLS = BN / 2;           // accumulator columns per epilogue warp
  static constexpr int STAGING_BYTES = 1024;        // per epilogue warp: 32 rows x 32 bytes
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_WARPS * STAGING_BYTES + 1024 + BAR_BYTES;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct GemmParams {
  int M, N, K;
  int num_m, num_n, num_kb;
  const float* alpha;
  const float* row_scale;
  const uint16_t* bias;
  void* D;
  int64_t ld_d;
  int out_f32;
  uint32_t* err;
};

// Output tile t -> (m block, n block), grouped 16 m-blocks at a time so that
// concurrently running CTAs share A and B panels in L2.
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
  constexpr int G = 16;
  const int per_group = G * num_n;
  const int g = t / per_group;
  const int first = g * G;
  const int gsz = min(G, num_m - first);
  const int r = t - g * per_group;
  mb = first + r % gsz;
  nb = r / gsz;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int KIND>
__global__ void __launch_bounds__(Cfg<KIND>::THREADS, 1)
    blockscaled_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                            const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
  using C = Cfg<KIND>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::EPI_WARPS * C::STAGING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, C::EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSFA);
    prefetch_tensormap(&tmSFB);
    prefetch_tensormap(&tmD);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int num_tiles = p.num_m * p.num_n;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p.num_m, p.num_n, mb, nb);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
          tma_load_2d(st, &tmA, &full[stage], kb * C::ROW_BYTES, mb * C::BM);
          tma_load_2d(st + C::A_BYTES, &tmB, &full[stage], kb * C::ROW_BYTES, nb * C::BN);
          tma_load_3d(st + C::A_BYTES + C::B_BYTES, &tmSFA, &full[stage], 0, kb * C::ATOMS, mb);
          tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, &full[stage], 0, kb * C::ATOMS, nb * 2);
          ++issued[stage];
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
      }
      // Every issued copy must have landed before the CTA may exit.
      for (int s = 0; s < C::STAGES; ++s)
        if (issued[s] && !mbar_wait(&full[s], (issued[s] - 1u) & 1u, nullptr)) raise_error(p.err, kErrTimeout);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
        if (!mbar_wait(acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sbase = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sfa_t = tmem + C::ACC_COLS + stage * C::SF_COLS;
          const uint32_t sfb_t = sfa_t + C::SFA_COLS;
          const uint32_t sfa_s = sbase + C::A_BYTES + C::B_BYTES;
          const uint32_t sfb_s = sfa_s + C::SFA_BYTES;
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a) tc_cp_32x128b_warpx4(sfa_t + 4 * a, desc_sf_block(sfa_s + 512 * a));
#pragma unroll
          for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int a = 0; a < C::ATOMS; ++a)
              tc_cp_32x128b_warpx4(sfb_t + 8 * a + 4 * rt, desc_sf_block(sfb_s + 512 * (rt * C::ATOMS + a)));
          const uint64_t adesc = desc_kmajor_sw128(sbase);
          const uint64_t bdesc = desc_kmajor_sw128(sbase + C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::MMAS; ++kk) {
            const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
            // 32 bytes of K per MMA: advance the start address by 32 >> 4.
            if constexpr (KIND == kNVF4)
              tc_mma_nvf4(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_nvf4(C::BM, C::BN), sfa_t + 4u * kk,
                          sfb_t + 8u * kk, accumulate);
            else
              tc_mma_mxf8(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc_mxf8(C::BM, C::BN, static_cast<uint32_t>(kk)),
                          sfa_t, sfb_t, accumulate);
          }
          tc_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
      }
      // No MMA may still be running when tensor memory is freed.
      tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) raise_error(p.err, kErrTimeout);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;               // 0..7
    const int q = warp & 3;                // tensor-memory lane quarter this warp may read
    const int half = ew >> 2;              // which 128 accumulator columns
    uint8_t* stage_buf = staging + ew * C::STAGING_BYTES;
    const float alpha = p.alpha ? __ldg(p.alpha) : 1.0f;
    // One staging row = 32 bytes = W output elements; the two 16-byte halves
    // are swapped on rows 4..7 of every 8 (TMA's 32-byte swizzle), which keeps
    // the 32 lanes' shared-memory writes at the minimum of 4 wavefronts.
    constexpr int W_BF16 = 16, W_F32 = 8;
    uint8_t* my_row = stage_buf + lane * 32;
    const uint32_t swz = (lane >> 2) & 1u;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(t, p.num_m, p.num_n, mb, nb);
      if (!mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag)) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after_sync();
      uint32_t acc[4][32];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * C::EPI_COLS);
#pragma unroll
      for (int k = 0; k < 4; ++k) tmem_ld_32cols(taddr + 32u * k, acc[k]);
      tmem_ld_wait();
      // accumulator is in registers: hand tensor memory back to the MMA warp
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);

      const int row0 = mb * C::BM + q * 32;
      const int row = row0 + static_cast<int>(lane);
      float scale = alpha;
      if (p.row_scale != nullptr && row < p.M) scale = __fmul_rn(alpha, __ldg(p.row_scale + row));
      const int col0 = nb * C::BN + half * C::EPI_COLS;
      if (p.out_f32) {
#pragma unroll
        for (int j = 0; j < C::EPI_COLS / W_F32; ++j) {
          const int n0 = col0 + j * W_F32;
          if (n0 >= p.N) break;
          float b[W_F32];
          uint4 bv = make_uint4(0u, 0u, 0u, 0u);
          if (p.bias != nullptr) bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n0));
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            b[2 * i] = bf16_bits_to_f32(bw[i] & 0xFFFFu);
            b[2 * i + 1] = bf16_bits_to_f32(bw[i] >> 16);
          }
          float y[W_F32];
#pragma unroll
          for (int i = 0; i < W_F32; ++i) {
            const int c = j * W_F32 + i;
            y[i] = __fmaf_rn(__uint_as_float(acc[c >> 5][c & 31]), scale, b[i]);
          }
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          *reinterpret_cast<float4*>(my_row + 16 * (0u ^ swz)) = make_float4(y[0], y[1], y[2], y[3]);
          *reinterpret_cast<float4*>(my_row + 16 * (1u ^ swz)) = make_float4(y[4], y[5], y[6], y[7]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmD, stage_buf, n0, row0);
            bulk_commit_group();
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < C::EPI_COLS / W_BF16; ++j) {
          const int n0 = col0 + j * W_BF16;
          if (n0 >= p.N) break;
          float b[W_BF16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint4 bv = make_uint4(0u, 0u, 0u, 0u);
            if (p.bias != nullptr && n0 + 8 * h < p.N) bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * h));
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              b[8 * h + 2 * i] = bf16_bits_to_f32(bw[i] & 0xFFFFu);
              b[8 * h + 2 * i + 1] = bf16_bits_to_f32(bw[i] >> 16);
            }
          }
          uint32_t packed[W_BF16 / 2];
#pragma unroll
          for (int i = 0; i < W_BF16 / 2; ++i) {
            const int c = j * W_BF16 + 2 * i;
            packed[i] = pack_bf16x2(__fmaf_rn(__uint_as_float(acc[c >> 5][c & 31]), scale, b[2 * i]),
                                    __fmaf_rn(__uint_as_float(acc[(c + 1) >> 5][(c + 1) & 31]), scale, b[2 * i + 1]));
          }
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          *reinterpret_cast<uint4*>(my_row + 16 * (0u ^ swz)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
          *reinterpret_cast<uint4*>(my_row + 16 * (1u ^ swz)) = make_uint4(packed[4], packed[5], packed[6], packed[7]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmD, stage_buf, n0, row0);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Row-major uint8 matrix [rows, row_bytes], boxes of box_rows x 128 bytes, 128-byte swizzle.
int encode_operand(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = encode_tiled_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_INVALID_ARG;
}

// Tile-mapped scale buffer viewed as [bands][tiles per band][512 bytes] with
// 8-byte elements; a box covers `atoms` consecutive 512-byte tiles of `bands`
// consecutive row bands.
int encode_scales(CUtensorMap* m, const void* base, int64_t bands, int64_t tiles_per_band, int atoms, int box_bands) {
  cuuint64_t dims[3] = {64u, static_cast<cuuint64_t>(tiles_per_band), static_cast<cuuint64_t>(bands)};
  cuuint64_t strides[2] = {512u, static_cast<cuuint64_t>(tiles_per_band * 512)};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(atoms), static_cast<cuuint32_t>(box_bands)};
  cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = encode_tiled_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(base), dims, strides, box, es,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_INVALID_ARG;
}

// Row-major output [rows, ld] of bf16 or fp32, boxes of 32 rows x 32 bytes, 32-byte swizzle.
int encode_output(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  const int64_t esize = f32 ? 4 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * esize)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(32 / esize), 32u};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = encode_tiled_fn()(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base,
                                 dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_INVALID_ARG;
}

template <int KIND>
int run_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
             int64_t K, const float* alpha, const float* row_scale, const uint16_t* bias, void* D, int d_dtype,
             int64_t ld_d, cudaStream_t stream) {
  using C = Cfg<KIND>;
  const int64_t group = KIND == kNVF4 ? 16 : 32;
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return BSP_ERR_INVALID_ARG;
  if (d_dtype != BSP_OUT_BF16 && d_dtype != BSP_OUT_F32) return BSP_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return BSP_OK;
  if (N % 8 != 0 || ld_d < N) return BSP_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return BSP_ERR_INVALID_ARG;
  if (!A || !B || !sfA || !sfB || !D) return BSP_ERR_INVALID_ARG;
  const int64_t esize = d_dtype == BSP_OUT_F32 ? 4 : 2;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfA) || !aligned16(sfB) || !aligned16(D) ||
      (bias && !aligned16(bias)) || (ld_d * esize) % 16 != 0 || (row_scale && (reinterpret_cast<uintptr_t>(row_scale) & 3u)) ||
      (alpha && (reinterpret_cast<uintptr_t>(alpha) & 3u)))
    return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (encode_tiled_fn() == nullptr) return BSP_ERR_CUDA;

  const int64_t row_bytes = KIND == kNVF4 ? K / 2 : K;
  const int64_t tiles_per_band = round_up(K / group, 4) / 4;
  CUtensorMap tmA, tmB, tmSFA, tmSFB, tmD;
  if ((st = encode_operand(&tmA, A, M, row_bytes, C::BM)) != BSP_OK) return st;
  if ((st = encode_operand(&tmB, B, N, row_bytes, C::BN)) != BSP_OK) return st;
  if ((st = encode_scales(&tmSFA, sfA, ceil_div(M, 128), tiles_per_band, C::ATOMS, 1)) != BSP_OK) return st;
  if ((st = encode_scales(&tmSFB, sfB, ceil_div(N, 128), tiles_per_band, C::ATOMS, 2)) != BSP_OK) return st;
  if ((st = encode_output(&tmD, D, M, N, ld_d, d_dtype == BSP_OUT_F32)) != BSP_OK) return st;

  static bool attr_set[64] = {};
  if (!attr_set[dev.id]) {
    if (cudaFuncSetAttribute(blockscaled_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return launch_status();
    attr_set[dev.id] = true;
  }

  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.num_m = static_cast<int>(ceil_div(M, C::BM));
  p.num_n = static_cast<int>(ceil_div(N, C::BN));
  p.num_kb = static_cast<int>(ceil_div(row_bytes, C::ROW_BYTES));
  p.alpha = alpha;
  p.row_scale = row_scale;
  p.bias = bias;
  p.D = D;
  p.ld_d = ld_d;
  p.out_f32 = d_dtype == BSP_OUT_F32;
  p.err = dev.err_word;
  const int64_t tiles = static_cast<int64_t>(p.num_m) * p.num_n;
  const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  blockscaled_gemm_kernel<KIND><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tmA, tmB, tmSFA, tmSFB, tmD, p);
  return launch_status();
}

}  // namespace
}  // namespace bsp

extern "C" {

int nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
               int64_t K, const float* alpha, const float* row_scale, const uint16_t* bias, void* D, int d_dtype,
               int64_t ld_d, bsp_stream_t stream) {
  return bsp::run_gemm<bsp::kNVF4>(A, sfA, B, sfB, M, N, K, alpha, row_scale, bias, D, d_dtype, ld_d, stream);
}

int mxfp8_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
               int64_t K, const float* alpha, const uint16_t* bias, void* D, int d_dtype, int64_t ld_d,
               bsp_stream_t stream) {
  return bsp::run_gemm<bsp::kMXF8>(A, sfA, B, sfB, M, N, K, alpha, nullptr, bias, D, d_dtype, ld_d, stream);
}

}  // extern "C"
