// fd_attn_tc.cuh — mask-free window attention on tcgen05 (sm_100a).
//
// Paper Sec. 3.3: the current frame's queries attend, with no mask, to every
// cached key of the window (itself plus W past frames). Keys of ring slot s
// are stored at rows [s*L, (s+1)*L) of the block's cache, so the window's keys
// are the contiguous range [win*L, (win + n_valid)*L) of the frame state
// (win = 0 except in a mirrored ring, where every slot is stored twice) and
// softmax, being invariant to the order of keys, needs no slot bookkeeping.
//
// One CTA = one head x 128 queries of one video stream (blockIdx.z; each
// stream has its own frame state and cache slab); 192 threads, 2 CTAs per SM.
// A launch may cover n_sub sub-frames of the paper head's refinement blocks
// at once: blockIdx.z / n_split = tau * B + b picks sub-frame tau of stream b,
// with its own frame state (and so its own key window in the shared ring).
// Keys are consumed in tiles of 64.
//   warp 0      TMA: Q once, then per stage K (64 keys x 64) and the
//               transposed V (64 dims x 64 keys)
//   warp 1      TMEM allocator; lane 0 issues S(j) = Q K_j^T (SS form) into
//               S buffer j mod 3 once O += P(j-3) V(j-3) has read that
//               buffer; lane 1 issues O += P(j) V_j (TS form: P read from
//               TMEM) as soon as P(j) is written, then releases the K/V stage.
//               Each lane's tcgen05.commit tracks only its own MMAs. Launches
//               with single_issuer set run both streams from lane 0 instead,
//               polling both hand-offs (same products, same order per stream)
//   warps 2..5  softmax, one query row per thread: S row from TMEM, base-2
//               online softmax with lazy rescaling (O is rescaled in TMEM only
//               when the running max grows by more than 2^8), P packed to bf16
//               and written over the S it came from. After the first tile, P
//               is formed against the running reference before the tile's
//               own max is known; the max (which only decides the rare
//               rescale, after which P is formed again) then overlaps the
//               exponentials instead of preceding them
// TMEM columns: S buffer b (b < 3) at 64 b, with P(j) in the first 32 columns
// of its buffer; O at 192. S runs up to three tiles ahead of the softmax,
// whose only synchronisation per tile is the wait for S(j) and the arrival
// that hands P(j) to the PV issuer. (Measured against two S buffers with
// separate P columns: bit-identical output, equal time at 1080p, 7% faster
// at 480p.) Keys past n_valid*L inside the last tile get probability 0.
//
// Key splitting (n_split > 1, for launches that fill the GPU's CTA slots
// poorly): the key tiles of every (query tile, head, stream) are divided into
// n_split contiguous ranges, one CTA each (blockIdx.z = stream * n_split +
// split). Each CTA writes its unnormalised O, running max and sum to scratch
// (part_o, part_ml), fences, and counts itself in counter[unit]; the CTA that
// arrives last combines the partials in split order (deterministic), writes O
// and resets the counter for the next launch. No CTA waits for another.
#pragma once

#include "fd_ptx.cuh"

namespace fd {

struct TcAttnParams {
  void* o;            // [n_sub][B][L][H*64] bf16
  int L, H, G;
  int B;              // video streams
  int n_sub;          // sub-frames per launch (1, or r_t for a whole refinement block)
  int layer;          // block index: cache map slab (layer * B + stream) * G + g
  int fs_stride;      // FrameStates per stream
  float scale_log2;   // log2(e) / sqrt(64)
  const FrameState* fs;  // state of stream b, sub-frame tau: fs[b * fs_stride + tau]
  int* status;
  // key splitting (n_split 1: off); unit = ((tau * B + b) * H + head) * gridDim.x + query tile
  int n_split;
  float* part_o;      // [unit][n_split][128][64] unnormalised O
  float* part_ml;     // [unit][n_split][128][2] running max (log2 domain), sum
  int* counter;       // [unit] CTAs of the unit done so far (0 between launches)
  // bounds of the bounds-checked build (FD_IN_BOUNDS)
  int kv_rows;        // rows of one (layer, stream, group) slab of the ring
  int n_slabs;        // slabs in the ring's tensor maps: layers x B x G
  int single_issuer;  // 1: one thread issues S and PV (else one lane each)
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
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

// D[tmem] (+)= A[tmem] * B[smem]^T (A: M rows in lanes, K packed 2 per column).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);      // a -> low half (lower k)
  return *reinterpret_cast<uint32_t*>(&v);
}

// p = 2^(s * sc - m) for one 64-key S row: packed bf16 pairs into pk[32];
// returns the row sum. Scores of masked keys are -inf and give exactly 0.
__device__ __forceinline__ float exp_pack64(const float* x, float sc, float m, uint32_t* pk) {
  const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(-m, -m);
  float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
  for (int c = 0; c < 64; c += 8) {
    float2 e0 = __ffma2_rn(make_float2(x[c], x[c + 1]), sc2, nm2);
    float2 e1 = __ffma2_rn(make_float2(x[c + 2], x[c + 3]), sc2, nm2);
    float2 e2 = __ffma2_rn(make_float2(x[c + 4], x[c + 5]), sc2, nm2);
    float2 e3 = __ffma2_rn(make_float2(x[c + 6], x[c + 7]), sc2, nm2);
    e0 = make_float2(ex2(e0.x), ex2(e0.y)); e1 = make_float2(ex2(e1.x), ex2(e1.y));
    e2 = make_float2(ex2(e2.x), ex2(e2.y)); e3 = make_float2(ex2(e3.x), ex2(e3.y));
    a0 = __fadd2_rn(a0, e0); a1 = __fadd2_rn(a1, e1);
    a2 = __fadd2_rn(a2, e2); a3 = __fadd2_rn(a3, e3);
    pk[c / 2 + 0] = pack_bf16(e0.x, e0.y); pk[c / 2 + 1] = pack_bf16(e1.x, e1.y);
    pk[c / 2 + 2] = pack_bf16(e2.x, e2.y); pk[c / 2 + 3] = pack_bf16(e3.x, e3.y);
  }
  a0 = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
  return a0.x + a0.y;
}

__device__ __forceinline__ float tile_max64(const float* x) {
  float m0 = max3(x[0], x[1], x[2]), m1 = max3(x[3], x[4], x[5]);
#pragma unroll
  for (int c = 6; c < 62; c += 4) { m0 = max3(m0, x[c], x[c + 1]); m1 = max3(m1, x[c + 2], x[c + 3]); }
  m0 = max3(m0, x[62], x[63]);
  return fmaxf(m0, m1);
}

struct TcAttnSmem {
  static constexpr int kStages = 4;
  static constexpr int kQ = 0;                                // 16 KB
  static constexpr int kKV = 16384;                           // stages x (K 8 KB + V^T 8 KB)
  static constexpr int kKVStage = 16384;
  static constexpr int kBar = kKV + kStages * kKVStage;
  // q_full, kv_full[ST], kv_empty[ST], s_full[3], p_full[3], p_free[3], o_final
  static constexpr int kNumBars = 1 + 2 * kStages + 10;
  static constexpr int kBytes = kBar + kNumBars * 8 + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr int kThreads = 192;
  static constexpr int kTmemCols = 256;
};

__global__ void __launch_bounds__(TcAttnSmem::kThreads, 2)
    tc_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, TcAttnParams p) {
  using S = TcAttnSmem;
  constexpr int ST = S::kStages;
  constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64);   // 128 queries x 64 keys
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, 64);   // 128 queries x 64 dims
  constexpr uint32_t kColO = 192;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + ST;
  uint64_t* s_full = kv_empty + ST;                 // [3]
  uint64_t* p_full = s_full + 3;                    // [3]
  uint64_t* p_free = p_full + 3;                    // [3]
  uint64_t* o_final = p_free + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * 128, h = blockIdx.y;
  const int bq = blockIdx.z / p.n_split, split = blockIdx.z - bq * p.n_split;
  const int bs = bq % p.B, tau = bq / p.B;            // video stream, sub-frame
  const int g = h / (p.H / p.G);
  const int lg = (p.layer * p.B + bs) * p.G + g;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int b = 0; b < 3; ++b) {
      mbar_init(&s_full[b], 1); mbar_init(&p_full[b], 128); mbar_init(&p_free[b], 1);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmQ); prefetch_tensormap(&tmK); prefetch_tensormap(&tmV);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, S::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();                                 // Q, K, V and the frame state
  griddep_launch();
  const FrameState& fst = p.fs[size_t(bs) * p.fs_stride + tau];
  int n_keys = fst.n_valid * p.L;
  const int key0 = fst.win * p.L;                 // first key row of the window
  if (!FD_IN_BOUNDS(key0 + n_keys <= p.kv_rows && lg < p.n_slabs && tau < p.n_sub, p.status))
    n_keys = 0;
  // the V^T tile's inner coordinate must be 16-byte aligned: a window start
  // off that grid (never produced by the host, which mirrors only rings with
  // L % 8 == 0) is refused rather than loaded
  if (key0 & 7) {
    if (threadIdx.x == 0) report_status(p.status, FD_ERR_BOUNDS);
    n_keys = 0;
  }
  const int n_kt_all = (n_keys + 63) / 64;
  // this CTA's key tiles: [j0, j0 + n_kt) (all of them without splitting)
  const int j0 = split * n_kt_all / p.n_split;
  const int n_kt = (split + 1) * n_kt_all / p.n_split - j0;

  if (warp == 0) {
    if (lane == 0) {                                       // ---- TMA producer
      mbar_arrive_expect_tx(q_full, 16384);
      tma_load_4d(smem + S::kQ, &tmQ, 0, q0, bq, h, q_full);
      for (int j = 0; j < n_kt; ++j) {
        const int st = j % ST;
        if (!mbar_wait(&kv_empty[st], ((j / ST) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* kv = smem + S::kKV + st * S::kKVStage;
        mbar_arrive_expect_tx(&kv_full[st], S::kKVStage);
        tma_load_3d(kv, &tmK, 0, key0 + (j0 + j) * 64, lg, &kv_full[st]);
        tma_load_3d(kv + 8192, &tmV, key0 + (j0 + j) * 64, 0, lg, &kv_full[st]);
      }
    }
  } else if (warp == 1) {
    if (p.single_issuer) {                                 // uniform per launch
      if (lane == 0) {                                     // ---- one issuer for S and PV
        // one thread polls both hand-offs, so neither MMA stream waits behind
        // the other lane's blocking wait in the same warp
        bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
        int js = 0, jp = 0;                                // next S tile, next PV tile
        unsigned long long t_idle = 0;
        while (ok && jp < n_kt) {
          bool progress = false;
          if (jp < js && mbar_try_wait(&p_full[jp % 3], (jp / 3) & 1)) {
            tc_fence_after();
            const uint32_t sv = smem_u32(smem + S::kKV + (jp % ST) * S::kKVStage + 8192);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_ts(tmem_base + kColO, tmem_base + 64 * (jp % 3) + 8 * k, sw128_desc(sv) + 2 * k,
                        kIdescO, (jp | k) != 0);
            tc_commit(&p_free[jp % 3]);
            tc_commit(&kv_empty[jp % ST]);
            ++jp;
            progress = true;
          }
          // S(js) once its stage is loaded and O += P(js-3) V(js-3) has read its buffer
          if (js < n_kt && js < jp + 3 && mbar_try_wait(&kv_full[js % ST], (js / ST) & 1) &&
              (js < 3 || mbar_try_wait(&p_free[js % 3], ((js / 3) - 1) & 1))) {
            tc_fence_after();
            const uint32_t sq = smem_u32(smem + S::kQ);
            const uint32_t sk = smem_u32(smem + S::kKV + (js % ST) * S::kKVStage);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma_ss(tmem_base + 64 * (js % 3), sw128_desc(sq) + 2 * k, sw128_desc(sk) + 2 * k,
                        kIdescS, k != 0);
            tc_commit(&s_full[js % 3]);
            ++js;
            progress = true;
          }
          if (progress) {
            t_idle = 0;
          } else if (*abort_flag) {
            ok = false;
          } else if (t_idle == 0) {
            t_idle = global_ns();
          } else if (global_ns() - t_idle > kWaitTimeoutNs) {   // bounded like mbar_wait
            *abort_flag = 1;
            report_status(p.status, FD_ERR_TIMEOUT);
            ok = false;
          }
        }
        if (ok) tc_commit(o_final);
      }
    } else if (lane == 0) {                                // ---- S issuer
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j < n_kt; ++j) {
        const int st = j % ST, b = j % 3;
        if (!mbar_wait(&kv_full[st], (j / ST) & 1, abort_flag, p.status)) break;
        // buffer b last held P(j-3): O += P(j-3) V(j-3) must have read it
        if (j >= 3 && !mbar_wait(&p_free[b], ((j / 3) - 1) & 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + S::kQ);
        const uint32_t sk = smem_u32(smem + S::kKV + st * S::kKVStage);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_ss(tmem_base + 64 * b, sw128_desc(sq) + 2 * k, sw128_desc(sk) + 2 * k, kIdescS,
                    k != 0);
        tc_commit(&s_full[b]);
      }
    } else if (lane == 1) {                                // ---- PV issuer
      bool ok = true;
      for (int i = 0; ok && i < n_kt; ++i) {
        const int b = i % 3;
        if (!mbar_wait(&p_full[b], (i / 3) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sv = smem_u32(smem + S::kKV + (i % ST) * S::kKVStage + 8192);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc_mma_ts(tmem_base + kColO, tmem_base + 64 * b + 8 * k, sw128_desc(sv) + 2 * k, kIdescO,
                    (i | k) != 0);
        tc_commit(&p_free[b]);
        tc_commit(&kv_empty[i % ST]);
      }
      if (ok) tc_commit(o_final);
    }
  } else {                                                 // ---- softmax warps
    const int quarter = warp & 3;                          // TMEM lanes 32*quarter ..
    const int r = quarter * 32 + lane;                     // query row within the tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tm_o = tmem_base + lane_off + kColO;
    const float sc = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int b = j % 3;
      if (!mbar_wait_warp(&s_full[b], (j / 3) & 1, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();
      float x[64];
      {
        uint32_t r0[32], r1[32];
        const uint32_t tm_s = tmem_base + lane_off + 64 * b;
        tmem_ld32(tm_s, r0); tmem_ld32(tm_s + 32, r1);
        tmem_ld_wait();
        reg_fence(r0); reg_fence(r1);
#pragma unroll
        for (int c = 0; c < 32; ++c) { x[c] = __uint_as_float(r0[c]); x[32 + c] = __uint_as_float(r1[c]); }
      }
      const int valid = n_keys - (j0 + j) * 64;            // keys of this tile in range
      if (valid < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = (c < valid) ? x[c] : -INFINITY;
        // P is 0 for those keys, and their V^T columns (a ring slot not yet
        // written since the reset, or the row padding) may hold anything: a
        // NaN there would still reach O as 0 x NaN, so zero them in the
        // stage before the PV product reads it. The stage's TMA load is
        // complete (its barrier phase cannot move on before P(j) arrives).
        const int st = j % ST;
        if (!mbar_wait_warp(&kv_full[st], (j / ST) & 1, abort_flag, p.status)) { ok = false; break; }
        uint8_t* vt = smem + S::kKV + st * S::kKVStage + 8192;   // [64 dims][128 B], 128-B swizzle
        const int t = threadIdx.x - 64, d = t >> 1;
        for (int c = valid + (t & 1); c < 64; c += 2)
          *reinterpret_cast<uint16_t*>(vt + d * 128 + (((c >> 3) ^ (d & 7)) << 4) + (c & 7) * 2) = 0;
        fence_proxy_async_smem();
      }
      uint32_t pk[32];
      float lt = 0.f, mx;
      if (j == 0) {
        mx = tile_max64(x) * sc;
        m_ref = mx;
        lt = exp_pack64(x, sc, m_ref, pk);
      } else {
        lt = exp_pack64(x, sc, m_ref, pk);           // independent of the tile max
        mx = tile_max64(x) * sc;
      }
      const bool rescale = j > 0 && mx > m_ref + 8.f;
      const float corr = rescale ? ex2(m_ref - mx) : 1.f;
      if (rescale) {                                 // rare: redo this row's P
        m_ref = mx;
        l *= corr;
        lt = exp_pack64(x, sc, m_ref, pk);
      }
      l += lt;
      if (__any_sync(0xffffffffu, rescale)) {
        // O *= corr (rare): every earlier O += P V must have landed first
        const int jp = j - 1;
        if (!mbar_wait_warp(&p_free[jp % 3], (jp / 3) & 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t o0[32], o1[32];
        tmem_ld32(tm_o, o0); tmem_ld32(tm_o + 32, o1);
        tmem_ld_wait();
        reg_fence(o0); reg_fence(o1);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          o0[c] = __float_as_uint(__uint_as_float(o0[c]) * corr);
          o1[c] = __float_as_uint(__uint_as_float(o1[c]) * corr);
        }
        tmem_st32(tm_o, o0); tmem_st32(tm_o + 32, o1);
      }
      tmem_st32(tmem_base + lane_off + 64 * b, pk);        // P over the S it came from
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    // the o_final commit is awaited even for an empty key range, so that no
    // asynchronous arrival can land after the CTA has exited
    const bool have_o = ok && mbar_wait_warp(o_final, 0, abort_flag, p.status);
    float v[64];
    if (have_o && n_kt > 0) {
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tm_o, o0); tmem_ld32(tm_o + 32, o1);
      tmem_ld_wait();
      reg_fence(o0); reg_fence(o1);
#pragma unroll
      for (int c = 0; c < 32; ++c) { v[c] = __uint_as_float(o0[c]); v[32 + c] = __uint_as_float(o1[c]); }
    } else {
#pragma unroll
      for (int c = 0; c < 64; ++c) v[c] = 0.f;
      m_ref = -INFINITY;
      l = 0.f;
    }
    const int row = q0 + r;
    if (p.n_split == 1) {
      if (have_o && row < p.L) {
        const float inv = 1.f / l;
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] *= inv;
        store_vec<bf16, 64>(static_cast<bf16*>(p.o) + (size_t(bq) * p.L + row) * p.H * 64 +
                                size_t(h) * 64, v);
      }
    } else if (FD_IN_BOUNDS(bq < p.B * p.n_sub && split < p.n_split, p.status)) {   // uniform per CTA
      // this key range's partial result
      const size_t unit = (size_t(bq) * p.H + h) * gridDim.x + blockIdx.x;
      const size_t prow = (unit * p.n_split + split) * 128 + r;
      float4* po = reinterpret_cast<float4*>(p.part_o + prow * 64);
#pragma unroll
      for (int c = 0; c < 16; ++c) po[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      reinterpret_cast<float2*>(p.part_ml)[prow] = make_float2(m_ref, l);
      __threadfence();
      asm volatile("bar.sync 1, 128;" ::: "memory");      // the four softmax warps
      if (threadIdx.x == 64) {
        const int done = atomicAdd(p.counter + unit, 1);
        const int last = done == p.n_split - 1;
        if (last) p.counter[unit] = 0;                    // ready for the next launch
        *last_flag = last;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (*last_flag) {
        __threadfence();
        // combine the n_split partials of this row in split order
        float mstar = -INFINITY;
        for (int sp = 0; sp < p.n_split; ++sp)
          mstar = fmaxf(mstar, reinterpret_cast<const float2*>(p.part_ml)[(unit * p.n_split + sp) * 128 + r].x);
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] = 0.f;
        for (int sp = 0; sp < p.n_split; ++sp) {
          const size_t q = (unit * p.n_split + sp) * 128 + r;
          const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml) + q);
          const float w = ex2(ml.x - mstar);              // 0 for an empty range
          lsum += w * ml.y;
          const float4* pq = reinterpret_cast<const float4*>(p.part_o + q * 64);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 t = __ldcg(pq + c);
            v[4 * c] += w * t.x; v[4 * c + 1] += w * t.y; v[4 * c + 2] += w * t.z; v[4 * c + 3] += w * t.w;
          }
        }
        if (row < p.L) {
          const float inv = 1.f / lsum;
#pragma unroll
          for (int c = 0; c < 64; ++c) v[c] *= inv;
          store_vec<bf16, 64>(static_cast<bf16*>(p.o) + (size_t(bq) * p.L + row) * p.H * 64 +
                                  size_t(h) * 64, v);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  drain_after_abort(abort_flag);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

}  // namespace fd
