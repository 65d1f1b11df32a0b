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
// Design (persistent, one CTA per SM, warp-specialised):
//   warp 0      TMA producer: per stage, the CTA's 128 rows of A and its rows
//               of B (128 bytes of K each, 128-byte swizzle) plus the matching
//               128x4 scale tiles, into shared memory; completion is counted on
//               the stage's mbarrier.
//   warp 1      MMA issuer (one thread): once a stage's data and scale factors
//               are ready, issues four block-scaled MMAs (K = 64 fp4 / 32 fp8
//               each) accumulating fp32 in tensor memory, and releases the
//               stage (tcgen05.commit).
//   warps 4-7   scale-factor warps, one per 32-lane quarter of tensor memory:
//               read the stage's 128x4 scale tiles from shared memory and write
//               them into the stage's scale columns of tensor memory
//               (tcgen05.st; each quarter holds the scales of all rows, which is
//               the replicated layout the block-scaled MMA reads).  Keeping the
//               scale traffic off the tensor pipe lets it overlap the MMAs of
//               the previous stages.
//   warps 8-15  epilogue, two warps per 32-lane quarter of tensor memory, each
//               owning half of the tile's accumulator columns: read all of them
//               into registers (tcgen05.ld), hand the accumulator back to the
//               MMA warp at once, then apply alpha, row scale and bias in fp32,
//               round once, stage 32 rows x 32 bytes in swizzled shared memory
//               and write them with TMA stores (full 32-byte sectors;
//               rows/columns past M/N clipped).
//   (roles by warp index: 0 producer, 1 MMA, 2-3 idle (relays in a pair
//   follower), 4-7 scales, 8-15 epilogue: four warpgroups, so that setmaxnreg
//   can move registers from the first two, which need few, to the epilogue's,
//   which holds a 128 x 128 half-accumulator per warpgroup)
// CTA pairs (CG = 2, large M): a cluster of two CTAs computes a 256 x 256
// tile with tcgen05.mma.cta_group::2.  Each CTA loads its 128 rows of A and
// 128 of the tile's 256 rows of B (the MMA reads both CTAs' shared memory and
// writes each CTA's 128 accumulator rows into its own tensor memory), and the
// scale tiles of all 256 rows of B, which each CTA's scale warps write into
// its own tensor memory.  Per SM that is 38 KB of operands per stage instead
// of 54 KB for the same MMA work, which is what sets the stage rate: the SMs
// take in operands from L2 more slowly than the tensor pipe consumes them.
// The leader (rank 0) issues the MMAs and multicasts its commits to both
// CTAs' barriers; the follower's scale and epilogue warps arrive on barriers
// of their own CTA, and its idle warps 2 and 3 relay each completed phase to
// the leader with one relaxed cluster-scope arrival (an arrival with
// cluster-scope release from the warps that had just written tensor memory
// took about 1 us under load).
// Output tiles are 128 x 256 with one accumulator (256 tensor-memory
// columns): two accumulators of 256 columns would leave no room for the stages'
// scale factors, and 128-column tiles with two accumulators measured slower (an
// N = 128 block-scaled MMA takes about as long to issue as an N = 256 one), so
// the next tile's MMAs wait until the epilogue has read the accumulator, which
// it does first thing.  When the 128 x 128 tiles of a GEMM fit in one wave
// (small M), the kernel is instantiated with BN = 128: twice the CTAs then
// stream the weight, which sets the time there.
// Tensor memory: the accumulator; then, per pipeline stage, the stage's
// scale factors (a scale column may only be rewritten once the stage's MMAs
// have completed, which the stage's empty barrier already guarantees).
// Ragged M / N / K edges: TMA fills out-of-range rows, K bytes and scale tiles
// with zeros (zero codes times zero scales add nothing); TMA stores clip.
// Every wait is bounded; a wait that runs out raises the device error word and
// the CTA drains its outstanding copies and MMAs, frees tensor memory and exits.
#include "bsp_device.cuh"
#include "bsp_internal.h"

// Tuning knobs (compile-time): pipeline depth, and how the epilogue writes D --
// 1: 32x32-byte swizzled shared-memory staging + TMA stores, with
// BSP_GEMM_STAGING_BUFS buffers per epilogue warp; 0: 16-byte stores straight
// from registers.
#ifndef BSP_GEMM_STAGES
#define BSP_GEMM_STAGES 8  // upper bound; the stages that fit shared and tensor memory are used
#endif
#ifndef BSP_GEMM_EPI_TMA
#define BSP_GEMM_EPI_TMA 1
#endif
#ifndef BSP_GEMM_STAGING_BUFS
#define BSP_GEMM_STAGING_BUFS 1
#endif
// Rasterisation: m-blocks per tile group; 0 chooses by operand size (see
// launch_gemm).
// Smallest M for which the main kernel runs as CTA pairs (cta_group::2).
#ifndef BSP_GEMM_PAIR_MIN_M
#define BSP_GEMM_PAIR_MIN_M 512
#endif
#ifndef BSP_GEMM_GROUP_M
#define BSP_GEMM_GROUP_M 0
#endif
// 1: output TMA stores carry an L2 evict-first hint.
#ifndef BSP_GEMM_STORE_EVICT_FIRST
#define BSP_GEMM_STORE_EVICT_FIRST 1
#endif
// Largest M for which the transposed skinny-M kernel is used (above it the
// main kernel with 128-column tiles streams the weight faster: M = 64,
// N = 13824, K = 5120 takes 12.0 against 14.4 us; at M = 48 the two are even).
// Activation scales in the 8x4 layout always take the skinny kernel, for
// M <= kSf8MaxM.
#ifndef BSP_GEMM_SKINNY_MAX_M
#define BSP_GEMM_SKINNY_MAX_M 48
#endif
// K bytes per operand row per pipeline stage of the NVFP4 main kernel (128 or
// 64; 64 halves the stage size and doubles the stage count).
#ifndef BSP_GEMM_NVF4_ROW_BYTES
#define BSP_GEMM_NVF4_ROW_BYTES 128
#endif

namespace bsp {
namespace {

enum Kind : int { kNVF4 = 0, kMXF8 = 1 };

constexpr int64_t kSf8MaxM = 64;  // rows of an activation whose scales may be in the 8x4 layout

constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int KIND, int BN_ = 256, int CG_ = 1>
struct Cfg {
  static constexpr int BM = 128;                        // accumulator rows (tensor-memory lanes) per CTA
  static constexpr int BN = BN_;                        // output tile columns (256, or 128 for few tiles)
  static constexpr int CG = CG_;                        // CTAs sharing one MMA (2: a CTA pair)
  static_assert(BN == 256 || BN == 128, "tile width");
  static_assert(CG == 1 || (CG == 2 && BN == 256), "CTA pairs take 256 x 256 tiles");
  static constexpr int TILE_M = BM * CG;                // output tile rows
  static constexpr int B_ROWS = BN / CG;                // rows of B each CTA loads
  static constexpr int ROW_BYTES = KIND == kNVF4 ? BSP_GEMM_NVF4_ROW_BYTES : 128;  // K bytes per row per stage
  static constexpr int MMAS = ROW_BYTES / 32;                                    // per stage, 32 bytes of K each
  static constexpr int ATOMS = KIND == kNVF4 ? ROW_BYTES / 32 : 1;  // 128x4 scale tiles per 128 rows per stage
  static_assert(ROW_BYTES == 128 || ROW_BYTES == 64, "stage row width");
  static constexpr int B_BANDS = BN / 128;              // 128-row bands of B per tile
  static constexpr int A_BYTES = BM * ROW_BYTES;
  static constexpr int B_BYTES = B_ROWS * ROW_BYTES;
  static constexpr int SFA_BYTES = ATOMS * 512;
  static constexpr int SFB_BYTES = B_BANDS * ATOMS * 512;  // the scales of all BN rows of B, in each CTA
  static constexpr int TX_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;  // per stage
  static constexpr int STAGE_BYTES = (TX_BYTES + 1023) / 1024 * 1024;
  static constexpr int SFA_COLS = ATOMS * 4;            // per stage, replicated layout
  static constexpr int SFB_COLS = ATOMS * 4 * B_BANDS;
  static constexpr int SF_COLS = SFA_COLS + SFB_COLS;   // 48 (fp4) / 12 (fp8)
  static constexpr int SFB_COLS_PER_MMA = KIND == kNVF4 ? 4 * B_BANDS : 0;  // fp8: one scale set per stage
  static constexpr int TMEM_COLS = 512;
  static constexpr int EPI_WARPS = 8;
  static constexpr int EPI_COLS = BN / 2;  // accumulator columns per epilogue warp
  static constexpr bool EPI_TMA = BSP_GEMM_EPI_TMA != 0;
  static constexpr int STAGING_BUFS = EPI_TMA ? BSP_GEMM_STAGING_BUFS : 0;
  static constexpr int STAGING_BYTES = 1024 * STAGING_BUFS;  // per epilogue warp: buffers of 32 rows x 32 bytes
  static constexpr int SF_WARPS = 4;
  // Four warpgroups: 0 = producer, MMA issuer and two idle warps; 1 = the
  // scale-factor warps; 2 and 3 = the epilogue.  Warpgroups 0 and 1 give up
  // registers (WG0_REGS, SF_REGS) so that the epilogue (EPI_REGS) can read the
  // whole accumulator into registers before handing it back to the MMA warp.
  static constexpr int FIRST_SF_WARP = 4;
  static constexpr int FIRST_EPI_WARP = 8;
  static constexpr int THREADS = 16 * 32;
  static constexpr int LAUNCH_REGS = 65536 / THREADS;  // 128
  static constexpr int WG0_REGS = 40, SF_REGS = 88, EPI_REGS = 192;
  static_assert(128 * (WG0_REGS + SF_REGS + 2 * EPI_REGS) == THREADS * LAUNCH_REGS, "register split");
  static constexpr int BAR_BYTES = 256;
  static constexpr int FIXED_BYTES = EPI_WARPS * STAGING_BYTES + 1024 + BAR_BYTES;
  static constexpr int ACC_COLS = BN;  // one fp32 accumulator
  static constexpr int STAGES = cmin(cmin((232448 - FIXED_BYTES) / STAGE_BYTES, (TMEM_COLS - ACC_COLS) / SF_COLS),
                                     BSP_GEMM_STAGES);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED_BYTES;
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(ACC_COLS + STAGES * SF_COLS <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(4 * STAGES + 4 <= BAR_BYTES / 8 - 1, "barrier space");
};

struct GemmParams {
  int M, N, K;
  int num_m, num_n, num_kb;
  int split;    // CTAs of a cluster sharing one output tile's K range (skinny kernel)
  int group_m;  // m-blocks per rasterisation group
  const float* alpha;
  const float* row_scale;
  const uint16_t* bias;
  void* D;
  int64_t ld_d;
  int out_f32;
  uint32_t* err;
};

// Output tile t -> (m block, n block), grouped G m-blocks at a time so that
// concurrently running CTAs share A and B panels in L2 (G is chosen on the host
// so that a group's A panel stays well inside L2 while B streams past it).
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int G, int& mb, int& nb) {
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

template <int KIND, int BN, int CG>
__global__ void __launch_bounds__(Cfg<KIND, BN, CG>::THREADS, 1)
    blockscaled_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                            const __grid_constant__ CUtensorMap tmD, const GemmParams p) {
  using C = Cfg<KIND, BN, CG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::EPI_WARPS * C::STAGING_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_ready = empty + C::STAGES;
  uint64_t* acc_full = sf_ready + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* sf_local = drain + 1;              // pair follower: its scale warps, per stage
  uint64_t* acc_local = sf_local + C::STAGES;  // pair follower: its epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_local + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  // CTA pair: rank 0 (the leader) issues the MMAs for both, and its commits
  // arrive on the barriers of both CTAs.  The follower's scale and epilogue
  // warps arrive on barriers of their own CTA; one of its idle warps forwards
  // each completed phase to the leader with a single cluster-scope arrival (a
  // cluster-scope release straight from the warps that wrote tensor memory
  // measured about 1 us per arrival).
  const uint32_t rank = C::CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0u;
  constexpr uint32_t kPeerArrivals = C::CG == 2 ? 1u : 0u;  // the follower's forwarded arrival

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], C::SF_WARPS + kPeerArrivals);
      mbar_init(&sf_local[s], C::SF_WARPS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, C::EPI_WARPS + kPeerArrivals);
    mbar_init(acc_local, C::EPI_WARPS);
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
    if constexpr (C::CG == 2) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  __syncwarp();
  if constexpr (C::CG == 2)
    cluster_sync();  // the peer's barriers are initialised before anything arrives on them
  else
    __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // Set-up above overlaps the previous kernel under programmatic launch; every
  // global access below comes after its completion.
  grid_dependency_wait();
  const int num_tiles = p.num_m * p.num_n;
  const int first_tile = static_cast<int>(blockIdx.x) / C::CG;
  const int tile_step = static_cast<int>(gridDim.x) / C::CG;

  if (warp < C::FIRST_SF_WARP) {
    // warpgroup 0: producer, MMA issuer, two idle warps
    regs_dec<C::WG0_REGS>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        uint32_t stage = 0, phase = 0;
        uint32_t issued[C::STAGES];
        for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
        bool ok = true;
        for (int t = first_tile; t < num_tiles && ok; t += tile_step) {
          int mb, nb;
          tile_coords(t, p.num_m, p.num_n, p.group_m, mb, nb);
          // this CTA's 128 rows of A and its share of B's rows (all of them,
          // or its half in a pair); the scales of all BN rows of B
          const int a_band = mb * C::CG + static_cast<int>(rank);
          const int b_row = nb * C::BN + static_cast<int>(rank) * C::B_ROWS;
          for (int kb = 0; kb < p.num_kb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + stage * C::STAGE_BYTES;
            mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
            tma_load_2d(st, &tmA, &full[stage], kb * C::ROW_BYTES, a_band * C::BM);
            tma_load_2d(st + C::A_BYTES, &tmB, &full[stage], kb * C::ROW_BYTES, b_row);
            tma_load_3d(st + C::A_BYTES + C::B_BYTES, &tmSFA, &full[stage], 0, kb * C::ATOMS, a_band);
            tma_load_3d(st + C::A_BYTES + C::B_BYTES + C::SFA_BYTES, &tmSFB, &full[stage], 0, kb * C::ATOMS,
                        nb * C::B_BANDS);
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
      if (lane == 0 && leader) {
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        int it = 0;
        constexpr uint16_t kPair = 0x3;  // commits arrive on the barriers of both CTAs of a pair
        auto commit = [&](uint64_t* bar) {
          if constexpr (C::CG == 2)
            tc_commit_pair(bar, kPair);
          else
            tc_commit(bar);
        };
        // barriers that the peer CTA arrives on are read with cluster-scope acquire
        auto wait_shared = [&](uint64_t* bar, uint32_t par) {
          if constexpr (C::CG == 2)
            return mbar_wait_cluster(bar, par, abort_flag);
          else
            return mbar_wait(bar, par, abort_flag);
        };
        for (int t = first_tile; t < num_tiles && ok; t += tile_step, ++it) {
          // the epilogue (of both CTAs) has read the previous tile's accumulator
          if (!wait_shared(acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          for (int kb = 0; kb < p.num_kb; ++kb) {
            // the scale warps (of both CTAs) signal after their stage landed and
            // its scales are in tensor memory
            if (!wait_shared(&sf_ready[stage], phase)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t sbase = smem_u32(smem + stage * C::STAGE_BYTES);
            const uint32_t sfa_t = tmem + C::ACC_COLS + stage * C::SF_COLS;
            const uint32_t sfb_t = sfa_t + C::SFA_COLS;
            const uint64_t adesc = desc_kmajor_swizzled(sbase, C::ROW_BYTES);
            const uint64_t bdesc = desc_kmajor_swizzled(sbase + C::A_BYTES, C::ROW_BYTES);
#pragma unroll
            for (int kk = 0; kk < C::MMAS; ++kk) {
              const uint32_t accumulate = (kb > 0 || kk > 0) ? 1u : 0u;
              // 32 bytes of K per MMA: advance the start address by 32 >> 4.
              if constexpr (KIND == kNVF4) {
                const uint32_t idesc = idesc_nvf4(C::TILE_M, C::BN);
                const uint32_t sfb_k = sfb_t + static_cast<uint32_t>(C::SFB_COLS_PER_MMA * kk);
                if constexpr (C::CG == 2)
                  tc_mma_nvf4_pair(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, sfa_t + 4u * kk, sfb_k, accumulate);
                else
                  tc_mma_nvf4(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, sfa_t + 4u * kk, sfb_k, accumulate);
              } else {
                const uint32_t idesc = idesc_mxf8(C::TILE_M, C::BN, static_cast<uint32_t>(kk));
                if constexpr (C::CG == 2)
                  tc_mma_mxf8_pair(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, sfa_t, sfb_t, accumulate);
                else
                  tc_mma_mxf8(tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, sfa_t, sfb_t, accumulate);
              }
            }
            commit(&empty[stage]);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          commit(acc_full);
        }
        if (!ok) {
          *abort_flag = 1u;
          raise_error(p.err, kErrTimeout);
        }
        // No MMA may still be running when tensor memory is freed.
        commit(drain);
        if (!mbar_wait(drain, 0u, nullptr)) raise_error(p.err, kErrTimeout);
      } else if (lane == 0) {
        // pair follower: its MMAs are issued by the leader, whose last commit
        // arrives here too
        if (!mbar_wait(drain, 0u, nullptr)) raise_error(p.err, kErrTimeout);
      }
    } else if (C::CG == 2 && !leader && lane == 0) {
      // pair follower, warp 2: each stage its scale warps complete, one
      // arrival on the leader's sf_ready; warp 3: each accumulator its
      // epilogue releases, one arrival on the leader's acc_empty
      bool ok = true;
      if (warp == 2) {
        const uint32_t peer = mapa_shared(smem_u32(sf_ready), 0u);
        uint32_t stage = 0, phase = 0;
        for (int t = first_tile; t < num_tiles && ok; t += tile_step) {
          for (int kb = 0; kb < p.num_kb; ++kb) {
            if (!mbar_wait(&sf_local[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_remote_relaxed(peer + 8u * stage);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      } else if (warp == 3) {
        const uint32_t peer = mapa_shared(smem_u32(acc_empty), 0u);
        int it = 0;
        for (int t = first_tile; t < num_tiles && ok; t += tile_step, ++it) {
          if (!mbar_wait(acc_local, static_cast<uint32_t>(it) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_remote_relaxed(peer);
        }
      }
      if (!ok) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
      }
    }
  } else if (warp < C::FIRST_EPI_WARP) {
    // ------------------------------------------------------------ scale factors (warpgroup 1)
    regs_dec<C::SF_REGS>();
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    uint64_t* sf_mine = leader ? sf_ready : sf_local;  // the follower's phases are forwarded
    for (int t = first_tile; t < num_tiles && ok; t += tile_step) {
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        // Line `lane` of each 512-byte scale tile (the scales of rows lane,
        // lane+32, lane+64, lane+96 for 4 K-groups) becomes 4 consecutive
        // columns of this lane; every lane quarter gets the same copy.  Per
        // MMA step: 4 columns of A scales, then 4 per 128-row band of B.
        const uint8_t* sfa_s = smem + stage * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES;
        const uint8_t* sfb_s = sfa_s + C::SFA_BYTES;
        uint32_t v[C::SF_COLS];
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          const uint4 w = *reinterpret_cast<const uint4*>(sfa_s + 512 * a + lane * 16);
          v[4 * a + 0] = w.x;
          v[4 * a + 1] = w.y;
          v[4 * a + 2] = w.z;
          v[4 * a + 3] = w.w;
        }
#pragma unroll
        for (int rt = 0; rt < C::B_BANDS; ++rt)
#pragma unroll
          for (int a = 0; a < C::ATOMS; ++a) {
            const uint4 w = *reinterpret_cast<const uint4*>(sfb_s + 512 * (rt * C::ATOMS + a) + lane * 16);
            constexpr int kPerAtom = 4 * C::B_BANDS;
            v[C::SFA_COLS + kPerAtom * a + 4 * rt + 0] = w.x;
            v[C::SFA_COLS + kPerAtom * a + 4 * rt + 1] = w.y;
            v[C::SFA_COLS + kPerAtom * a + 4 * rt + 2] = w.z;
            v[C::SFA_COLS + kPerAtom * a + 4 * rt + 3] = w.w;
          }
        const uint32_t taddr = tmem + lane_base + C::ACC_COLS + stage * C::SF_COLS;
        if constexpr (C::SF_COLS == 48) {
          tmem_st_16cols(taddr, v);
          tmem_st_16cols(taddr + 16, v + 16);
          tmem_st_16cols(taddr + 32, v + 32);
        } else if constexpr (C::SF_COLS == 32) {
          tmem_st_16cols(taddr, v);
          tmem_st_16cols(taddr + 16, v + 16);
        } else if constexpr (C::SF_COLS == 24) {
          tmem_st_16cols(taddr, v);
          tmem_st_8cols(taddr + 16, v + 16);
        } else if constexpr (C::SF_COLS == 12) {
          tmem_st_4cols(taddr, v);
          tmem_st_8cols(taddr + 4, v + 4);
        } else {
          static_assert(C::SF_COLS == 8, "scale columns per stage");
          tmem_st_8cols(taddr, v);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_mine[stage]);
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
  } else {
    // ------------------------------------------------------------ epilogue (warpgroups 2 and 3)
    regs_inc<C::EPI_REGS>();
    const int ew = warp - C::FIRST_EPI_WARP;  // 0..7
    const int q = warp & 3;    // tensor-memory lane quarter this warp may read
    const int half = ew >> 2;  // which half of the tile's columns
    uint8_t* stage_buf = staging + ew * C::STAGING_BYTES;
    const float alpha = p.alpha ? __ldg(p.alpha) : 1.0f;
    // One staging row = 32 bytes = W output elements; the two 16-byte halves
    // are swapped on rows 4..7 of every 8 (TMA's 32-byte swizzle), which keeps
    // the 32 lanes' shared-memory writes at the minimum of 4 wavefronts.
    constexpr int W_BF16 = 16, W_F32 = 8;
    const uint32_t swz = (lane >> 2) & 1u;
    uint32_t store_seq = 0;  // TMA stores issued by this warp (picks the staging buffer)
    const uint64_t evict_first = l2_policy_evict_first();

    // Writes 32 bytes of this lane's row into the staging buffer, then one
    // lane stores the 32 x 32-byte box at (n0, row0).
    auto stage_and_store = [&](int n0, int row0, uint4 lo, uint4 hi) {
      if constexpr (C::EPI_TMA) {
        uint8_t* buf = stage_buf + (store_seq % C::STAGING_BUFS) * 1024;
        if (lane == 0) bulk_wait_read_allow<C::STAGING_BUFS - 1>();
        __syncwarp();
        *reinterpret_cast<uint4*>(buf + lane * 32 + 16 * (0u ^ swz)) = lo;
        *reinterpret_cast<uint4*>(buf + lane * 32 + 16 * (1u ^ swz)) = hi;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (BSP_GEMM_STORE_EVICT_FIRST)
            tma_store_2d_hint(&tmD, buf, n0, row0, evict_first);
          else
            tma_store_2d(&tmD, buf, n0, row0);
          bulk_commit_group();
        }
        ++store_seq;
      } else {
        const int row = row0 + static_cast<int>(lane);
        if (row < p.M) {
          const int64_t esize = p.out_f32 ? 4 : 2;
          uint8_t* dst = static_cast<uint8_t*>(p.D) + (static_cast<int64_t>(row) * p.ld_d + n0) * esize;
          *reinterpret_cast<uint4*>(dst) = lo;
          if (n0 + 16 / esize < p.N) *reinterpret_cast<uint4*>(dst + 16) = hi;
        }
      }
    };

    uint64_t* acc_mine = leader ? acc_empty : acc_local;  // the follower's releases are forwarded
    auto release_accumulator = [&]() {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_mine);
    };

    int it = 0;
    for (int t = first_tile; t < num_tiles; t += tile_step, ++it) {
      int mb, nb;
      tile_coords(t, p.num_m, p.num_n, p.group_m, mb, nb);
      // Row scale and bias are fetched before the accumulator is ready.  The
      // bias of this warp's columns is spread over the lanes, four columns each
      // (lane j: columns col0 + 4j .. 4j + 3), and handed to every lane by
      // shuffles while the accumulator is read.
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(half * C::EPI_COLS);
      const int row0 = mb * C::TILE_M + static_cast<int>(rank) * C::BM + q * 32;
      const int row = row0 + static_cast<int>(lane);
      float scale = alpha;
      if (p.row_scale != nullptr && row < p.M) scale = __fmul_rn(alpha, __ldg(p.row_scale + row));
      const int col0 = nb * C::BN + half * C::EPI_COLS;
      uint2 bias4 = make_uint2(0u, 0u);
      if (p.bias != nullptr && col0 + 4 * static_cast<int>(lane) < p.N)
        bias4 = __ldg(reinterpret_cast<const uint2*>(p.bias + col0 + 4 * static_cast<int>(lane)));
      const bool got = C::CG == 2 ? mbar_wait_cluster(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag)
                                  : mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag);
      if (!got) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after_sync();

      if (!p.out_f32) {
        // bf16: read all of this warp's columns into registers and hand the
        // accumulator back at once (the next tile's MMAs start while this
        // one's epilogue arithmetic runs), then apply alpha, row scale and
        // bias, pack, and store from registers.
        uint32_t r[C::EPI_COLS];
#pragma unroll
        for (int c = 0; c < C::EPI_COLS / 32; ++c)
          tmem_ld_32cols(taddr + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(r + 32 * c));
        tmem_ld_wait();
        release_accumulator();
        uint32_t packed[C::EPI_COLS / 2];
#pragma unroll
        for (int c = 0; c < C::EPI_COLS / 32; ++c) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            // columns 32c + 2i, 2i + 1 are held by lane 8c + i/2
            const uint32_t bw = __shfl_sync(0xFFFFFFFFu, (i & 1) ? bias4.y : bias4.x, 8 * c + (i >> 1));
            packed[16 * c + i] =
                pack_bf16x2(__fmaf_rn(__uint_as_float(r[32 * c + 2 * i]), scale, bf16_bits_to_f32(bw & 0xFFFFu)),
                            __fmaf_rn(__uint_as_float(r[32 * c + 2 * i + 1]), scale, bf16_bits_to_f32(bw >> 16)));
          }
        }
#pragma unroll
        for (int j = 0; j < C::EPI_COLS / W_BF16; ++j) {
          const int n0 = col0 + j * W_BF16;
          if (n0 >= p.N) break;
          stage_and_store(n0, row0, make_uint4(packed[8 * j], packed[8 * j + 1], packed[8 * j + 2], packed[8 * j + 3]),
                          make_uint4(packed[8 * j + 4], packed[8 * j + 5], packed[8 * j + 6], packed[8 * j + 7]));
        }
      } else {
        // fp32: 16 columns at a time, tensor memory released at the end.
#pragma unroll 1
        for (int k = 0; k < C::EPI_COLS / 16; ++k) {
          uint32_t r[16];
          tmem_ld_16cols(taddr + 16u * k, r);
          tmem_ld_wait();
          const int nk = col0 + 16 * k;
          if (nk >= p.N) continue;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int n0 = nk + W_F32 * h;
            if (n0 >= p.N) break;
            uint4 bv = make_uint4(0u, 0u, 0u, 0u);
            if (p.bias != nullptr) bv = __ldg(reinterpret_cast<const uint4*>(p.bias + n0));
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            float y[W_F32];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              y[2 * i] = __fmaf_rn(__uint_as_float(r[8 * h + 2 * i]), scale, bf16_bits_to_f32(bw[i] & 0xFFFFu));
              y[2 * i + 1] = __fmaf_rn(__uint_as_float(r[8 * h + 2 * i + 1]), scale, bf16_bits_to_f32(bw[i] >> 16));
            }
            stage_and_store(n0, row0,
                            make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                                       __float_as_uint(y[3])),
                            make_uint4(__float_as_uint(y[4]), __float_as_uint(y[5]), __float_as_uint(y[6]),
                                       __float_as_uint(y[7])));
          }
        }
        release_accumulator();
      }
    }
    if constexpr (C::EPI_TMA) {
      if (lane == 0) bulk_wait_all();
    }
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncwarp();
  if constexpr (C::CG == 2)
    cluster_sync();  // no CTA of the pair leaves while the other may still signal it
  else
    __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    if constexpr (C::CG == 2)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Skinny M (M <= BSP_GEMM_SKINNY_MAX_M, and M <= 64 with 8x4 activation
// scales; e.g. per-token decode-like batches against a large weight): the GEMM
// is bound by streaming the weight from HBM, so it is run transposed,
// D^T = B A^T.  The weight is the MMA's 128-row operand (tiles of 128 weight
// rows, so ~N/128 CTAs stream disjoint weight panels through a deep pipeline of
// small stages) and the BNA <= 128 activation rows are the MMA's N side.  Same roles as the main kernel: warp 0 producer, warp 1 MMA issuer,
// warps 2-5 scale factors, warps 6-9 epilogue (lane = output column n, one
// TMEM column per activation row m; each warp writes 32 consecutive n of a
// row of D per instruction).
// ---------------------------------------------------------------------------
// kSf8: the activation scales are in the 8x4 layout (32-byte tiles of 8 rows x
// 4 K-groups, row-major); a stage's box is the BNA/8 row tiles x 4 K-group
// tiles (fp4) of 32 bytes.
// kSplit: the tile's K range is split over the CTAs of a thread-block cluster
// (split-K); each keeps its fp32 partial in a shared-memory buffer of
// 128 x (BNA + 4) floats (padded rows), and the cluster's rank 0 adds the
// others' partials, in rank order, through distributed shared memory.
template <int KIND, int BNA, bool kSf8 = false, bool kSplit = false>
struct SkCfg {
  static constexpr int BM = 128;                         // weight rows per tile (MMA M)
  static constexpr int ROW_BYTES = 128;
  static constexpr int MMAS = 4;
  static constexpr int ATOMS = KIND == kNVF4 ? 4 : 1;
  static constexpr int W_BYTES = BM * ROW_BYTES;
  static constexpr int X_BYTES = BNA * ROW_BYTES;
  static constexpr int SFW_BYTES = ATOMS * 512;
  static constexpr int SFX_BYTES = kSf8 ? (BNA / 8) * ATOMS * 32  // BNA/8 row tiles x ATOMS tiles of 32 bytes
                                        : ATOMS * 512;            // one 128-row band of activation scales
  static constexpr int TX_BYTES = W_BYTES + X_BYTES + SFW_BYTES + SFX_BYTES;
  static constexpr int STAGE_BYTES = (TX_BYTES + 1023) / 1024 * 1024;
  static constexpr int SFW_COLS = ATOMS * 4;
  static constexpr int SFX_COLS = ATOMS * 4;            // N <= 128: one column group per K step
  static constexpr int SF_COLS = SFW_COLS + SFX_COLS;
  static constexpr int ACC_COLS = BNA;
  static constexpr int TMEM_COLS = 512;
  static constexpr int SF_WARPS = 4, EPI_WARPS = 4;
  static constexpr int THREADS = 64 + (SF_WARPS + EPI_WARPS) * 32;
  static constexpr int RED_STRIDE = BNA + 4;  // floats per partial row (one row per output column n)
  static constexpr int RED_BYTES = kSplit ? 128 * RED_STRIDE * 4 : 0;
  static constexpr int FIXED_BYTES = 1024 + 256 + RED_BYTES;
  static constexpr int STAGES =
      cmin(cmin((232448 - FIXED_BYTES) / STAGE_BYTES, (TMEM_COLS - ACC_COLS) / SF_COLS), 8);
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED_BYTES;
  static_assert(STAGES >= 2 && ACC_COLS + STAGES * SF_COLS <= TMEM_COLS, "budget");
};

template <int KIND, int BNA, bool kSf8, bool kSplit>
__global__ void __launch_bounds__(SkCfg<KIND, BNA, kSf8, kSplit>::THREADS, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmSFW, const __grid_constant__ CUtensorMap tmSFX,
                       const GemmParams p) {
  using C = SkCfg<KIND, BNA, kSf8, kSplit>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);  // split-K partial (kSplit)
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES + C::RED_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* sf_ready = empty + C::STAGES;
  uint64_t* acc_full = sf_ready + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* part_ready = drain + 1;  // rank 0: the other ranks' partials of the tile are in their buffers
  uint64_t* part_free = part_ready + 1;  // rank > 0: rank 0 has read this CTA's partial
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(part_free + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  // split-K: cluster rank r takes k-blocks [kb0, kb1) of every tile of its cluster
  const int S = kSplit ? p.split : 1;
  const uint32_t rank = kSplit ? cluster_ctarank() : 0u;
  const int kb0 = static_cast<int>(static_cast<int64_t>(p.num_kb) * rank / S);
  const int kb1 = static_cast<int>(static_cast<int64_t>(p.num_kb) * (rank + 1) / S);
  const int first_tile = static_cast<int>(blockIdx.x) / S, tile_step = static_cast<int>(gridDim.x) / S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], C::SF_WARPS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, C::EPI_WARPS);
    mbar_init(drain, 1);
    if constexpr (kSplit) {
      mbar_init(part_ready, static_cast<uint32_t>((S - 1) * C::EPI_WARPS * 32));
      mbar_init(part_free, C::EPI_WARPS * 32);
    }
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmSFW);
    prefetch_tensormap(&tmSFX);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  if constexpr (kSplit) cluster_sync();  // every CTA's barriers exist before another CTA arrives on them
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();  // as in the main kernel
  // tile t: weight panel nb = t % num_n (fastest), activation block mb = t / num_n
  const int num_tiles = p.num_m * p.num_n;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued[C::STAGES];
      for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
      bool ok = true;
      for (int t = first_tile; t < num_tiles && ok; t += tile_step) {
        const int nb = t % p.num_n, mb = t / p.num_n;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
          tma_load_2d(st, &tmW, &full[stage], kb * C::ROW_BYTES, nb * C::BM);
          tma_load_2d(st + C::W_BYTES, &tmX, &full[stage], kb * C::ROW_BYTES, mb * BNA);
          tma_load_3d(st + C::W_BYTES + C::X_BYTES, &tmSFW, &full[stage], 0, kb * C::ATOMS, nb);
          if constexpr (kSf8)
            tma_load_2d(st + C::W_BYTES + C::X_BYTES + C::SFW_BYTES, &tmSFX, &full[stage], kb * C::ATOMS * 32,
                        mb * (BNA / 8));
          else
            tma_load_3d(st + C::W_BYTES + C::X_BYTES + C::SFW_BYTES, &tmSFX, &full[stage], 0, kb * C::ATOMS,
                        (mb * BNA) >> 7);
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
      for (int s = 0; s < C::STAGES; ++s)
        if (issued[s] && !mbar_wait(&full[s], (issued[s] - 1u) & 1u, nullptr)) raise_error(p.err, kErrTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = first_tile; t < num_tiles && ok; t += tile_step, ++it) {
        if (!mbar_wait(acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&sf_ready[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sbase = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t sfw_t = tmem + C::ACC_COLS + stage * C::SF_COLS;
          const uint32_t sfx_t = sfw_t + C::SFW_COLS;
          const uint64_t wdesc = desc_kmajor_sw128(sbase);
          const uint64_t xdesc = desc_kmajor_sw128(sbase + C::W_BYTES);
#pragma unroll
          for (int kk = 0; kk < C::MMAS; ++kk) {
            const uint32_t accumulate = (kb > kb0 || kk > 0) ? 1u : 0u;
            if constexpr (KIND == kNVF4)
              tc_mma_nvf4(tmem, wdesc + 2u * kk, xdesc + 2u * kk, idesc_nvf4(C::BM, BNA), sfw_t + 4u * kk,
                          sfx_t + 4u * kk, accumulate);
            else
              tc_mma_mxf8(tmem, wdesc + 2u * kk, xdesc + 2u * kk, idesc_mxf8(C::BM, BNA, static_cast<uint32_t>(kk)),
                          sfw_t, sfx_t, accumulate);
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
      tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) raise_error(p.err, kErrTimeout);
    }
  } else if (warp < 2 + C::SF_WARPS) {
    // scale warps: stage tiles -> replicated scale columns (see the main kernel)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int t = first_tile; t < num_tiles && ok; t += tile_step) {
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* sfw_s = smem + stage * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES;
        const uint8_t* sfx_s = sfw_s + C::SFW_BYTES;
        uint32_t v[C::SF_COLS];
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          const uint4 w = *reinterpret_cast<const uint4*>(sfw_s + 512 * a + lane * 16);
          uint4 x;
          if constexpr (kSf8) {
            // the 4 scales of activation row m for K-group tile a; rows past BNA are not in the box
            uint32_t q[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int m = static_cast<int>(lane) + 32 * j;
              if (m < BNA) q[j] = *reinterpret_cast<const uint32_t*>(sfx_s + (m >> 3) * (C::ATOMS * 32) + a * 32 +
                                                                      (m & 7) * 4);
            }
            x = make_uint4(q[0], q[1], q[2], q[3]);
          } else {
            x = *reinterpret_cast<const uint4*>(sfx_s + 512 * a + lane * 16);
          }
          v[4 * a + 0] = w.x;
          v[4 * a + 1] = w.y;
          v[4 * a + 2] = w.z;
          v[4 * a + 3] = w.w;
          v[C::SFW_COLS + 4 * a + 0] = x.x;
          v[C::SFW_COLS + 4 * a + 1] = x.y;
          v[C::SFW_COLS + 4 * a + 2] = x.z;
          v[C::SFW_COLS + 4 * a + 3] = x.w;
        }
        const uint32_t taddr = tmem + lane_base + C::ACC_COLS + stage * C::SF_COLS;
        if constexpr (C::SF_COLS == 32) {
          tmem_st_16cols(taddr, v);
          tmem_st_16cols(taddr + 16, v + 16);
        } else {
          static_assert(C::SF_COLS == 8, "scale columns per stage");
          tmem_st_8cols(taddr, v);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[stage]);
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
  } else {
    // epilogue: lane = output column n, TMEM column c = activation row m
    const int q = warp & 3;
    const float alpha = p.alpha ? __ldg(p.alpha) : 1.0f;
    const int nl = q * 32 + static_cast<int>(lane);  // output column within the panel
    float* my_red = red + nl * C::RED_STRIDE;
    int it = 0;
    for (int t = first_tile; t < num_tiles; t += tile_step, ++it) {
      const int nb = t % p.num_n, mb = t / p.num_n;
      const int n = nb * C::BM + nl;
      const bool n_ok = n < p.N;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      if (kSplit && rank != 0) {
        // split-K partial of ranks > 0: into this CTA's buffer, once rank 0
        // has read the previous tile's partial from it
        if (it > 0 && !mbar_wait_cluster(part_free, static_cast<uint32_t>(it - 1) & 1u, abort_flag)) {
          *abort_flag = 1u;
          raise_error(p.err, kErrTimeout);
          break;
        }
        if (!mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag)) {
          *abort_flag = 1u;
          raise_error(p.err, kErrTimeout);
          break;
        }
        tc_fence_after_sync();
#pragma unroll
        for (int c0 = 0; c0 < BNA; c0 += 16) {
          if (mb * BNA + c0 >= p.M) break;  // warp-uniform
          uint32_t r[16];
          tmem_ld_16cols(taddr + static_cast<uint32_t>(c0), r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4*>(my_red + c0 + 4 * j) =
                make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                            __uint_as_float(r[4 * j + 3]));
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        mbar_arrive_remote(mapa_shared(smem_u32(part_ready), 0u));  // every lane, after its own writes
        continue;
      }
      float b = 0.0f;
      if (p.bias != nullptr && n_ok) b = bf16_bits_to_f32(p.bias[n]);
      // alpha x row scale of this tile's activation rows, one row per lane,
      // fetched before the accumulator is ready and handed out by shuffles
      float rs[(BNA + 31) / 32];
#pragma unroll
      for (int j = 0; j < (BNA + 31) / 32; ++j) {
        const int m = mb * BNA + 32 * j + static_cast<int>(lane);
        rs[j] = (p.row_scale != nullptr && m < p.M) ? __fmul_rn(alpha, __ldg(p.row_scale + m)) : alpha;
      }
      if (!mbar_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag)) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
        break;
      }
      if (kSplit && !mbar_wait_cluster(part_ready, static_cast<uint32_t>(it) & 1u, abort_flag)) {
        *abort_flag = 1u;
        raise_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after_sync();
#pragma unroll
      for (int c0 = 0; c0 < BNA; c0 += 16) {
        if (mb * BNA + c0 >= p.M) break;  // warp-uniform
        uint32_t r[16];
        tmem_ld_16cols(taddr + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = __uint_as_float(r[i]);
        if constexpr (kSplit) {
          // the other ranks' partials, added in rank order (the sum does not
          // depend on which CTA finished first)
          for (int s = 1; s < S; ++s) {
            const uint32_t peer = mapa_shared(smem_u32(my_red + c0), static_cast<uint32_t>(s));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 v = ld_shared_cluster_f4(peer + 16u * j);
              acc[4 * j] = __fadd_rn(acc[4 * j], v.x);
              acc[4 * j + 1] = __fadd_rn(acc[4 * j + 1], v.y);
              acc[4 * j + 2] = __fadd_rn(acc[4 * j + 2], v.z);
              acc[4 * j + 3] = __fadd_rn(acc[4 * j + 3], v.w);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = mb * BNA + c0 + i;
          if (m >= p.M) break;  // warp-uniform
          const float scale = __shfl_sync(0xFFFFFFFFu, rs[(c0 + i) >> 5], (c0 + i) & 31);
          const float y = __fmaf_rn(acc[i], scale, b);
          if (n_ok) {
            if (p.out_f32)
              static_cast<float*>(p.D)[static_cast<int64_t>(m) * p.ld_d + n] = y;
            else
              static_cast<__nv_bfloat16*>(p.D)[static_cast<int64_t>(m) * p.ld_d + n] = __float2bfloat16_rn(y);
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      if constexpr (kSplit) {
        // the partials are read: each rank may reuse its buffer
        for (int s = 1; s < S; ++s) mbar_arrive_remote(mapa_shared(smem_u32(part_free), static_cast<uint32_t>(s)));
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  // no CTA leaves while another may still read its buffer or arrive on its barriers
  if constexpr (kSplit) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int encode_operand(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows,
                   int box_bytes = 128);
int encode_scales(CUtensorMap* m, const void* base, int64_t bands, int64_t tiles_per_band, int atoms, int box_bands);
int encode_rows_plain(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows, int box_bytes);

template <int KIND, int BNA, bool kSf8 = false, bool kSplit = false>
int launch_skinny(const DeviceInfo& dev, const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                  int64_t row_bytes, int64_t tiles_per_band, GemmParams p, cudaStream_t stream) {
  using C = SkCfg<KIND, BNA, kSf8, kSplit>;
  auto kernel = skinny_gemm_kernel<KIND, BNA, kSf8, kSplit>;
  static bool attr_set[64] = {};
  if (!attr_set[dev.id]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return launch_status();
    attr_set[dev.id] = true;
  }
  CUtensorMap tmW, tmX, tmSFW, tmSFX;
  int st;
  if ((st = encode_operand(&tmW, B, p.N, row_bytes, C::BM)) != BSP_OK) return st;
  if ((st = encode_operand(&tmX, A, p.M, row_bytes, BNA)) != BSP_OK) return st;
  if ((st = encode_scales(&tmSFW, sfB, ceil_div(p.N, 128), tiles_per_band, C::ATOMS, 1)) != BSP_OK) return st;
  if constexpr (kSf8) {
    // [row tiles][tiles_per_band x 32 bytes], boxes of BNA/8 row tiles x ATOMS tiles
    if ((st = encode_rows_plain(&tmSFX, sfA, ceil_div(p.M, 8), tiles_per_band * 32, BNA / 8, C::ATOMS * 32)) !=
        BSP_OK)
      return st;
  } else {
    if ((st = encode_scales(&tmSFX, sfA, ceil_div(p.M, 128), tiles_per_band, C::ATOMS, 1)) != BSP_OK) return st;
  }
  p.num_n = static_cast<int>(ceil_div(p.N, C::BM));
  p.num_m = static_cast<int>(ceil_div(p.M, BNA));
  if (!kSplit) p.split = 1;
  const int64_t tiles = static_cast<int64_t>(p.num_m) * p.num_n;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as in launch_gemm
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int64_t clusters = tiles < dev.sm_count / p.split ? tiles : dev.sm_count / p.split;
  if constexpr (kSplit) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(p.split);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    // no more clusters than are resident at once (a cluster's CTAs share one
    // GPC): the grid is one wave of them, each looping over its tiles
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * p.split), 1, 1);
    int resident = 0;
    if (cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg) != cudaSuccess) return launch_status();
    if (resident < 1) return BSP_ERR_CUDA;  // a cluster of this size does not fit: nothing launched
    if (clusters > resident) clusters = resident;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(clusters * p.split), 1, 1);
  if (cudaLaunchKernelEx(&cfg, kernel, tmW, tmX, tmSFW, tmSFX, p) != cudaSuccess) return launch_status();
  return launch_status();
}

// CTAs per tile of the skinny kernel: 1, or a split of K over a cluster of up
// to 4 CTAs when the tiles alone would leave at least half of the SMs without
// work (few weight panels: N <= ~9K) and every rank keeps at least 16 k-blocks
// (4096 fp4 elements of K): below that the cluster's start-up and reduction
// cost more than the extra streams gain (measured: K = 13824 gains 1.5x at
// S = 3, K = 5120 gains nothing, K = 1536 loses).
int skinny_split(const DeviceInfo& dev, int64_t tiles, int num_kb) {
  if (tiles * 2 > dev.sm_count) return 1;
  int64_t s = dev.sm_count / tiles;
  s = s < 4 ? s : 4;
  s = s < num_kb / 16 ? s : num_kb / 16;
  return s < 1 ? 1 : static_cast<int>(s);
}

template <int KIND, int BNA, bool kSf8 = false>
int launch_skinny_any(const DeviceInfo& dev, const uint8_t* A, const uint8_t* sfA, const uint8_t* B,
                      const uint8_t* sfB, int64_t row_bytes, int64_t tiles_per_band, GemmParams p,
                      cudaStream_t stream) {
  const int64_t tiles = ceil_div(p.N, 128) * ceil_div(p.M, BNA);
  p.split = skinny_split(dev, tiles, p.num_kb);
  if (p.split > 1)
    return launch_skinny<KIND, BNA, kSf8, true>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
  return launch_skinny<KIND, BNA, kSf8, false>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
}

// Row-major uint8 matrix [rows, row_bytes], boxes of box_rows x box_bytes (128
// or 64) with the matching TMA swizzle.
int encode_operand(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows, int box_bytes) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = encode_tiled_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_INVALID_ARG;
}

// Row-major bytes [rows, row_bytes], boxes of box_rows x box_bytes, no swizzle.
int encode_rows_plain(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows, int box_bytes) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = encode_tiled_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
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

template <int KIND, int BN, int CG = 1>
int launch_gemm(const DeviceInfo& dev, const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB,
                int64_t row_bytes, int64_t tiles_per_band, const CUtensorMap& tmD, GemmParams p,
                cudaStream_t stream) {
  using C = Cfg<KIND, BN, CG>;
  CUtensorMap tmA, tmB, tmSFA, tmSFB;
  int st;
  if ((st = encode_operand(&tmA, A, p.M, row_bytes, C::BM, C::ROW_BYTES)) != BSP_OK) return st;
  if ((st = encode_operand(&tmB, B, p.N, row_bytes, C::B_ROWS, C::ROW_BYTES)) != BSP_OK) return st;
  if ((st = encode_scales(&tmSFA, sfA, ceil_div(p.M, 128), tiles_per_band, C::ATOMS, 1)) != BSP_OK) return st;
  if ((st = encode_scales(&tmSFB, sfB, ceil_div(p.N, 128), tiles_per_band, C::ATOMS, C::B_BANDS)) != BSP_OK)
    return st;
  p.num_kb = static_cast<int>(ceil_div(row_bytes, C::ROW_BYTES));
  auto kernel = blockscaled_gemm_kernel<KIND, BN, CG>;
  static bool attr_set[64] = {};
  if (!attr_set[dev.id]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return launch_status();
    attr_set[dev.id] = true;
  }
  p.num_m = static_cast<int>(ceil_div(p.M, C::TILE_M));
  p.num_n = static_cast<int>(ceil_div(p.N, C::BN));
  const int64_t tiles = static_cast<int64_t>(p.num_m) * p.num_n;
  // one CTA (or CTA pair) per SM (pair of SMs), each looping over its tiles
  int64_t groups = dev.sm_count / CG;
  if (tiles < groups) groups = tiles;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  // programmatic launch: the kernel's set-up overlaps the previous kernel's tail
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (CG == 2) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    cfg.gridDim = dim3(static_cast<unsigned>(groups * 2), 1, 1);
    int resident = 0;  // no more pairs than are resident at once
    if (cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg) != cudaSuccess) return launch_status();
    if (resident < 1) return BSP_ERR_CUDA;  // a pair does not fit: nothing launched
    if (groups > resident) groups = resident;
  }
  const int ctas = static_cast<int>(groups * CG);
  cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
  if (BSP_GEMM_GROUP_M > 0) {
    p.group_m = BSP_GEMM_GROUP_M < p.num_m ? BSP_GEMM_GROUP_M : p.num_m;
  } else {
    // B (codes and scales) well inside L2: group just enough m-blocks that the
    // CTAs running at once cover every n-block, so each A panel is read from
    // DRAM once.  Large B: about 24 MiB of A per group, so the group's A panel
    // stays in L2 while B streams past it once per group.
    const int64_t b_bytes = static_cast<int64_t>(p.N) * row_bytes * 17 / 16;
    int64_t g;
    if (b_bytes < (32ll << 20)) {
      g = ceil_div(2ll * groups, p.num_n);
    } else {
      const int64_t a_panel = static_cast<int64_t>(C::TILE_M) * row_bytes * 17 / 16;
      g = (24ll << 20) / (a_panel > 0 ? a_panel : 1);
    }
    g = g < 8 ? 8 : g;
    p.group_m = static_cast<int>(g < p.num_m ? g : p.num_m);
  }
  if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmSFA, tmSFB, tmD, p) != cudaSuccess) return launch_status();
  return launch_status();
}

template <int KIND>
int run_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
             int64_t K, const float* alpha, const float* row_scale, const uint16_t* bias, void* D, int d_dtype,
             int64_t ld_d, cudaStream_t stream, int a_sf_layout = BSP_SF_LAYOUT_128X4) {
  const int64_t group = KIND == kNVF4 ? 16 : 32;
  if (M < 0 || N < 0 || K <= 0 || K % 32 != 0) return BSP_ERR_INVALID_ARG;
  if (d_dtype != BSP_OUT_BF16 && d_dtype != BSP_OUT_F32) return BSP_ERR_INVALID_ARG;
  const bool sf8 = a_sf_layout == BSP_SF_LAYOUT_8X4;
  if (!sf8 && a_sf_layout != BSP_SF_LAYOUT_128X4) return BSP_ERR_INVALID_ARG;
  if (sf8 && (KIND != kNVF4 || M > kSf8MaxM)) return BSP_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return BSP_OK;
  if (N % 8 != 0 || ld_d < N) return BSP_ERR_INVALID_ARG;
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30)) return BSP_ERR_INVALID_ARG;
  if (!A || !B || !sfA || !sfB || !D) return BSP_ERR_INVALID_ARG;
  const int64_t esize = d_dtype == BSP_OUT_F32 ? 4 : 2;
  if (!aligned16(A) || !aligned16(B) || !aligned16(sfA) || !aligned16(sfB) || !aligned16(D) ||
      (bias && !aligned16(bias)) || (ld_d * esize) % 16 != 0 ||
      (row_scale && (reinterpret_cast<uintptr_t>(row_scale) & 3u)) || (alpha && (reinterpret_cast<uintptr_t>(alpha) & 3u)))
    return BSP_ERR_ALIGNMENT;
  DeviceInfo dev;
  int st = current_device(&dev);
  if (st != BSP_OK) return st;
  if (encode_tiled_fn() == nullptr) return BSP_ERR_CUDA;

  const bool skinny = M <= BSP_GEMM_SKINNY_MAX_M;
  const int64_t row_bytes = KIND == kNVF4 ? K / 2 : K;
  const int64_t tiles_per_band = round_up(K / group, 4) / 4;
  CUtensorMap tmD;
  if ((st = encode_output(&tmD, D, M, N, ld_d, d_dtype == BSP_OUT_F32)) != BSP_OK) return st;

  GemmParams p;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.num_kb = static_cast<int>(ceil_div(row_bytes, 128));
  p.split = 1;
  p.alpha = alpha;
  p.row_scale = row_scale;
  p.bias = bias;
  p.D = D;
  p.ld_d = ld_d;
  p.out_f32 = d_dtype == BSP_OUT_F32;
  p.err = dev.err_word;
  if constexpr (KIND == kNVF4) {
    if (sf8) {  // 8x4 activation scales: M <= 64, the transposed kernel
      if (M <= 16) return launch_skinny_any<KIND, 16, true>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
      if (M <= 32) return launch_skinny_any<KIND, 32, true>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
      return launch_skinny_any<KIND, 64, true>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
    }
  }
  if (skinny) {
    if (M <= 16) return launch_skinny_any<KIND, 16>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
    if (M <= 32) return launch_skinny_any<KIND, 32>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
    if (M <= 64) return launch_skinny_any<KIND, 64>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
    return launch_skinny_any<KIND, 128>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, p, stream);
  }
  // 128-column tiles when they still fit in one wave: twice the CTAs stream B
  // (for small M the weight stream, not the tensor pipe, sets the time)
  if (ceil_div(M, 128) * ceil_div(N, 128) <= dev.sm_count)
    return launch_gemm<KIND, 128>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, tmD, p, stream);
  // many tiles: CTA pairs with 256 x 256 tiles, half of B per SM
  if (M >= BSP_GEMM_PAIR_MIN_M)
    return launch_gemm<KIND, 256, 2>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, tmD, p, stream);
  return launch_gemm<KIND, 256>(dev, A, sfA, B, sfB, row_bytes, tiles_per_band, tmD, p, stream);
}

}  // namespace
}  // namespace bsp

extern "C" {

int nvfp4_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
               int64_t K, const float* alpha, const float* row_scale, const uint16_t* bias, void* D, int d_dtype,
               int64_t ld_d, bsp_stream_t stream) {
  return bsp::run_gemm<bsp::kNVF4>(A, sfA, B, sfB, M, N, K, alpha, row_scale, bias, D, d_dtype, ld_d, stream);
}

int nvfp4_gemm_ex(const uint8_t* A, const uint8_t* sfA, int a_sf_layout, const uint8_t* B, const uint8_t* sfB,
                  int64_t M, int64_t N, int64_t K, const float* alpha, const float* row_scale, const uint16_t* bias,
                  void* D, int d_dtype, int64_t ld_d, bsp_stream_t stream) {
  return bsp::run_gemm<bsp::kNVF4>(A, sfA, B, sfB, M, N, K, alpha, row_scale, bias, D, d_dtype, ld_d, stream,
                                   a_sf_layout);
}

int mxfp8_gemm(const uint8_t* A, const uint8_t* sfA, const uint8_t* B, const uint8_t* sfB, int64_t M, int64_t N,
               int64_t K, const float* alpha, const uint16_t* bias, void* D, int d_dtype, int64_t ld_d,
               bsp_stream_t stream) {
  return bsp::run_gemm<bsp::kMXF8>(A, sfA, B, sfB, M, N, K, alpha, nullptr, bias, D, d_dtype, ld_d, stream);
}

}  // extern "C"
