// fd_gemm_tc.cuh — persistent tcgen05 GEMM with fused epilogues (sm_100a).
//
//   C[M][N] = A[M][K] * B[N][K]^T     A, B bf16 (K contiguous), fp32 accumulate
//                                     (F8: A, B FP8 E4M3, kind::f8f6f4)
//
// Used for every dense contraction of the FlashDecoder block (QKV, output
// projection, both MLP layers) and the final projection. Structure:
//   warp 0      TMA producer: A tile 128 x 128 bytes and B tile BN x 128 bytes
//               per stage (64 bf16 or 128 E4M3 of K), 128-byte swizzle, one
//               mbarrier (expect_tx) per stage
//   warp 1      TMEM allocator; lane 0 issues tcgen05.mma (M=128, N=BN,
//               32 bytes of K per instruction, 4 per stage) and commits
//   warps 2..   epilogue: tcgen05.ld of the 128 x BN fp32 accumulator, one
//               token row per thread, fused epilogue (fd_epilogue.cuh). The
//               GELU epilogues are arithmetic-bound and get 8 warps (two per
//               TMEM lane quarter, alternate 64-column chunks; measured 10%
//               faster); the others wait on memory and keep 4 (8 measured no
//               faster, and the QKV epilogue would spill)
// The accumulator is double-buffered in TMEM (2 x BN columns) so the
// epilogue of tile i overlaps the main loop of tile i+1. Tiles are handed out
// round-robin over a grid of at most one CTA per SM. Rows past M are read as
// zeros by TMA and never stored.
#pragma once

#include "fd_epilogue.cuh"
#include "fd_ptx.cuh"

namespace fd {

__host__ __device__ constexpr bool epi_resid(int kind) {
  return kind == EPI_RESID || kind == EPI_RESID_Q;
}

template <int BN, int STAGES, int KIND = EPI_QKV>
struct TcGemmSmem {
  static constexpr int kATile = 128 * 64 * 2;        // bytes
  static constexpr int kBTile = BN * 64 * 2;
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kBarOff = STAGES * kStage;
  // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], tmem slot, abort
  static constexpr int kEpiOff = kBarOff + (2 * STAGES + 4) * 8 + 16;
  // residual epilogues: per epilogue warp a [32 rows][36] fp32 transpose tile;
  // QKV: per epilogue warp a [32 rows][72] bf16 tile
  static constexpr int kEpiBytes = epi_resid(KIND) ? 4 * 32 * kResidPitch * 4
                                   : KIND == EPI_QKV ? 4 * 32 * kQkvPitch * 2 : 0;
  static constexpr int kBytes = kEpiOff + kEpiBytes;
  static constexpr int kAlloc = kBytes + 1024;        // slack for 1024-B alignment
};

__host__ __device__ constexpr int gemm_epi_threads(int kind) {
  return (kind == EPI_GELU || kind == EPI_GELU_Q) ? 256 : 128;
}
__host__ __device__ constexpr int gemm_threads(int kind) { return 64 + gemm_epi_threads(kind); }

template <int BN, int STAGES, int KIND, int DH, bool F8 = false>
__global__ void __launch_bounds__(gemm_threads(KIND), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   int K, EpiParams ep, int* status) {
  using S = TcGemmSmem<BN, STAGES, KIND>;
  constexpr int kEpiThreads = gemm_epi_threads(KIND);
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  constexpr uint32_t kTmemCols = 2 * BN;              // power of two: 128, 256 or 512
  static_assert((kTmemCols & (kTmemCols - 1)) == 0, "TMEM columns must be a power of 2");
  constexpr uint32_t kIdesc = F8 ? idesc_e4m3_f32(128, BN) : idesc_bf16_f32(128, BN);
  constexpr int kBK = F8 ? 128 : 64;                  // K elements per stage (128 bytes)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = ep.M;
  const int n_m = (M + 127) / 128, n_n = ep.N / BN;
  const int n_tiles = n_m * n_n, k_blocks = K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], kEpiThreads); }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();                                     // inputs of the previous kernel
  griddep_launch();

  if (warp == 0) {
    if (lane == 0) {                                  // ---- TMA producer
      int stage = 0; uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int m_blk = tile / n_n, n_blk = tile - (tile / n_n) * n_n;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, status)) goto producer_done;
          uint8_t* sa = smem + stage * S::kStage;
          mbar_arrive_expect_tx(&full[stage], S::kStage);
          tma_load_2d(sa, &tmA, kb * kBK, m_blk * 128, &full[stage]);
          tma_load_2d(sa + S::kATile, &tmB, kb * kBK, n_blk * BN, &full[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {                                  // ---- MMA issuer
      int stage = 0; uint32_t phase = 0; int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&acc_empty[buf], acc_phase ^ 1, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        bool ok = true;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * S::kStage);
          const uint64_t adesc = sw128_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + S::kATile);
#pragma unroll
          for (int k = 0; k < 4; ++k) {     // 32 bytes of K = 2 descriptor units
            if constexpr (F8)
              tc_mma_ss_f8(d_tmem, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0);
            else
              tc_mma_ss(d_tmem, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0);
          }
          tc_commit(&empty[stage]);         // stage reusable once these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);          // accumulator ready for the epilogue
      }
    }
  } else {                                            // ---- epilogue warps
    // kEpiThreads / 128 warps per TMEM lane quarter, alternate 64-column chunks
    constexpr int kPerQuarter = kEpiThreads / 128;
    const int quarter = warp & 3;                     // TMEM lanes 32*quarter ..
    const int half = (warp - 2) >> 2;
    int it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++it) {
      const int m_blk = tile / n_n, n_blk = tile - (tile / n_n) * n_n;
      const int buf = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // the RMSNorm row scale does not depend on the accumulator: its loads
      // overlap the tile's main loop
      const int row = m_blk * 128 + quarter * 32 + lane;
      float rs = 1.f;
      if (epi_normed(KIND) && row < M && ep.ssq) rs = row_scale(ep, row);
      if (!mbar_wait_warp(&acc_full[buf], acc_phase, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(quarter * 32) << 16) + buf * BN;
#pragma unroll 1
      for (int c = 64 * half; c < BN; c += 64 * kPerQuarter) {
        uint32_t r0[32], r1[32];
        tmem_ld32(taddr + c, r0);
        tmem_ld32(taddr + c + 32, r1);
        tmem_ld_wait();
        reg_fence(r0);
        reg_fence(r1);
        float acc[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) { acc[i] = __uint_as_float(r0[i]); acc[32 + i] = __uint_as_float(r1[i]); }
        if constexpr (epi_resid(KIND)) {
          // whole warp: rows m_blk*128 + 32*quarter .. +31 through a transpose tile
          float* tile = reinterpret_cast<float*>(smem + S::kEpiOff) + quarter * 32 * kResidPitch;
          resid_epilogue64<KIND, bf16>(ep, m_blk * 128 + quarter * 32, n_blk * BN + c, acc, tile, lane);
        } else if constexpr (KIND == EPI_QKV) {
          bf16* tile = reinterpret_cast<bf16*>(smem + S::kEpiOff) + quarter * 32 * kQkvPitch;
          qkv_epilogue64(ep, row, n_blk * BN + c, acc, rs, tile, lane);
        } else {
          if (row < M) epilogue64<KIND, bf16, DH>(ep, row, n_blk * BN + c, acc, rs);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  drain_after_abort(abort_flag);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace fd
