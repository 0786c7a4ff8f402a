// fd_attn_tc.cuh — mask-free window attention on tcgen05 (sm_100a).
//
// Paper Sec. 3.3: the current frame's queries attend, with no mask, to every
// cached key of the window (itself plus W past frames). Keys of ring slot s
// are stored at rows [s*L, (s+1)*L) of the block's cache, so the valid keys
// are always the contiguous range [0, n_valid*L) and softmax, being
// invariant to the order of keys, needs no slot bookkeeping.
//
// One CTA = one head x 128 queries, 192 threads:
//   warp 0      TMA: the Q tile once, then K (128 keys x 64) and the
//               transposed V (64 x 128 keys, as two 64-key halves) per stage
//   warp 1      TMEM allocator; lane 0 issues S_j = Q K_j^T into one of two
//               TMEM S buffers, then O += P_{j-1} V_{j-1} (software pipelined
//               so the tensor core works on S_j while the softmax runs on
//               S_{j-1})
//   warps 2..5  softmax, one query row per thread: S row from TMEM, base-2
//               online softmax with lazy rescaling (O is rescaled in TMEM
//               only when the running max grows by more than 2^8), P as bf16
//               into a 128-byte-swizzled shared tile, final O / l to global
// Keys past n_valid*L inside the last tile get probability 0.
#pragma once

#include "fd_ptx.cuh"

namespace fd {

struct TcAttnParams {
  void* o;            // [L][H*64] bf16
  int L, H, G;
  int layer;          // block index: third coordinate base of the cache maps
  float scale_log2;   // log2(e) / sqrt(64)
  const FrameState* fs;
  int* status;
};

constexpr int kAttnStages = 3;
struct TcAttnSmem {
  static constexpr int kQ = 0;                       // 128 x 64 bf16 = 16 KB
  static constexpr int kKV = 16384;                  // stages x (K 16 KB + V 16 KB)
  static constexpr int kKVStage = 32768;
  static constexpr int kP = kKV + kAttnStages * kKVStage;   // 2 x 32 KB
  static constexpr int kBar = kP + 2 * 32768;
  // q_full, kv_full[ST], kv_empty[ST], s_full[2], s_free[2], p_full[2], p_free[2], o_final
  static constexpr int kNumBars = 1 + 2 * kAttnStages + 8 + 1;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(192, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, TcAttnParams p) {
  using S = TcAttnSmem;
  constexpr int ST = kAttnStages;
  constexpr uint32_t kTmemCols = 512;                  // S0 [0,128) S1 [128,256) O [256,320)
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128);
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, 64);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + ST;
  uint64_t* s_full = kv_empty + ST;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* p_free = p_full + 2;
  uint64_t* o_final = p_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * 128, h = blockIdx.y;
  const int g = h / (p.H / p.G);
  const int lg = p.layer * p.G + g;
  const int n_keys = p.fs->n_valid * p.L;
  const int n_kt = (n_keys + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1); mbar_init(&s_free[b], 128);
      mbar_init(&p_full[b], 128); mbar_init(&p_free[b], 1);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmQ); prefetch_tensormap(&tmK); prefetch_tensormap(&tmV);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_o = tmem_base + 256;

  if (warp == 0) {
    if (lane == 0) {                                       // ---- TMA producer
      mbar_arrive_expect_tx(q_full, 16384);
      tma_load_3d(smem + S::kQ, &tmQ, 0, q0, h, q_full);
      for (int j = 0; j < n_kt; ++j) {
        const int st = j % ST;
        const uint32_t ph = (j / ST) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1, abort_flag, p.status)) break;
        uint8_t* kv = smem + S::kKV + st * S::kKVStage;
        mbar_arrive_expect_tx(&kv_full[st], S::kKVStage);
        tma_load_3d(kv, &tmK, 0, j * 128, lg, &kv_full[st]);
        tma_load_3d(kv + 16384, &tmV, j * 128, 0, lg, &kv_full[st]);
        tma_load_3d(kv + 16384 + 8192, &tmV, j * 128 + 64, 0, lg, &kv_full[st]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {                                       // ---- MMA issuer
      const uint32_t sq = smem_u32(smem + S::kQ);
      auto issue_pv = [&](int i) -> bool {
        const int b = i & 1, st = i % ST;
        if (!mbar_wait(&p_full[b], (i >> 1) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t sp = smem_u32(smem + S::kP + b * 32768);
        const uint32_t sv = smem_u32(smem + S::kKV + st * S::kKVStage + 16384);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int half = k >> 2, kk = k & 3;
          tc_mma_ss(tmem_o, sw128_desc(sp + half * 16384) + 2 * kk,
                    sw128_desc(sv + half * 8192) + 2 * kk, kIdescO, (i | k) != 0);
        }
        tc_commit(&p_free[b]);
        tc_commit(&kv_empty[st]);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j < n_kt; ++j) {
        const int st = j % ST, b = j & 1;
        if (!mbar_wait(&kv_full[st], (j / ST) & 1, abort_flag, p.status)) { ok = false; break; }
        if (!mbar_wait(&s_free[b], ((j >> 1) & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + S::kKV + st * S::kKVStage);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_ss(tmem_base + b * 128, sw128_desc(sq) + 2 * k, sw128_desc(sk) + 2 * k, kIdescS,
                    k != 0);
        tc_commit(&s_full[b]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(n_kt - 1)) tc_commit(o_final);
    }
  } else {                                                 // ---- softmax warps 2..5
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                     // query row within the tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int b = j & 1;
      if (!mbar_wait_warp(&s_full[b], (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      float x[128];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        const uint32_t ta = tmem_base + lane_off + b * 128;
        tmem_ld32(ta, r0); tmem_ld32(ta + 32, r1); tmem_ld32(ta + 64, r2); tmem_ld32(ta + 96, r3);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = __uint_as_float(r0[c]); x[32 + c] = __uint_as_float(r1[c]);
          x[64 + c] = __uint_as_float(r2[c]); x[96 + c] = __uint_as_float(r3[c]);
        }
      }
      tc_fence_before();
      mbar_arrive(&s_free[b]);
      const int valid = n_keys - j * 128;                  // keys of this tile in range
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        x[c] = (c < valid) ? x[c] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, x[c]);
      }
      if (j == 0) {
        m_ref = mx;
      } else if (mx > m_ref + 8.f) {
        // rescale O and l to the new reference max; O must hold P_{j-1} V_{j-1}
        if (!mbar_wait_warp(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const float corr = ex2(m_ref - mx);
        m_ref = mx;
        l *= corr;
        uint32_t o0[32], o1[32];
        tmem_ld32(tmem_o + lane_off, o0); tmem_ld32(tmem_o + lane_off + 32, o1);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          o0[c] = __float_as_uint(__uint_as_float(o0[c]) * corr);
          o1[c] = __float_as_uint(__uint_as_float(o1[c]) * corr);
        }
        tmem_st32(tmem_o + lane_off, o0); tmem_st32(tmem_o + lane_off + 32, o1);
        tmem_st_wait();
      }
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) { x[c] = ex2(x[c] - m_ref); rowsum += x[c]; }
      l += rowsum;
      // P buffer b was last read by the MMA of tile j-2
      if (j >= 2 && !mbar_wait_warp(&p_free[b], ((j - 2) >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
      uint8_t* prow = smem + S::kP + b * 32768 + r * 128;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const float* v = x + half * 64 + ch * 8;
          uint4 u;
          u.x = pack_bf16(v[0], v[1]); u.y = pack_bf16(v[2], v[3]);
          u.z = pack_bf16(v[4], v[5]); u.w = pack_bf16(v[6], v[7]);
          *reinterpret_cast<uint4*>(prow + half * 16384 + ((ch ^ (r & 7)) << 4)) = u;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && mbar_wait_warp(o_final, 0, abort_flag, p.status)) {
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tmem_o + lane_off, o0); tmem_ld32(tmem_o + lane_off + 32, o1);
      tmem_ld_wait();
      const int row = q0 + r;
      if (row < p.L) {
        const float inv = 1.f / l;
        float v[64];
#pragma unroll
        for (int c = 0; c < 32; ++c) { v[c] = __uint_as_float(o0[c]) * inv; v[32 + c] = __uint_as_float(o1[c]) * inv; }
        store_vec<bf16, 64>(static_cast<bf16*>(p.o) + size_t(row) * p.H * 64 + size_t(h) * 64, v);
      }
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
