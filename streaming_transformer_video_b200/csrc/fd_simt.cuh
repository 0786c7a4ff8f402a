// fd_simt.cuh — CUDA-core kernels of the FlashDecoder step:
//   step_begin   per-frame state from the device frame counter
//   embed        patchify gather + latent projection (paper Eq. 1), K = C' p^2
//                is tiny so this is a bandwidth-bound CUDA-core kernel
//   simt_gemm    fp32 GEMM + fused epilogue      (fp32 configuration)
//   simt_attn    fp32 unmasked window attention  (fp32 configuration)
// The fp32 configuration's tolerance (1e-4 absolute) rules out bf16/tf32
// tensor-core arithmetic, so its contractions run on CUDA cores.
#pragma once

#include "fd_epilogue.cuh"
#include "fd_ptx.cuh"

namespace fd {

// ---------------------------------------------------------------- step_begin
// B video streams, each with its own counter ctr[b] and 1 + n_sub states
// fs[b (1 + n_sub) + k]:
//   k = 0: latent frame t = ctr[b] in the backbone ring of W+1 frames;
//   k = 1 + tau, tau < n_sub (paper head, n_sub = r_t): sub-frame t r_t + tau
//   of the refinement ring (paper Sec. 3.4, Step 2), whose window is the last
//   r_t (W+1) sub-frames.
// A frame with absolute index t in a ring of `cap` slots and a window of
// `wnd` frames gets slot = t mod cap, n_valid = min(t, wnd - 1) + 1, and
// temporal RoPE angles t * theta^(-2m/d_t) (inv_freq[m], fp64 from the host)
// reduced mod 2 pi in fp64, so they stay exact for any stream length.
// The refinement ring either has cap = wnd slots (the window is every valid
// slot, win = 0), or, when all r_t sub-frames of a latent frame go through a
// refinement block in one launch (sub_mirror = 1), cap = r_t (W+2) - 1 slots
// stored twice (slot s at frame rows s and s + cap): writing a latent frame's
// r_t sub-frames then overwrites no slot that an earlier sub-frame of the same
// frame still attends to, and each sub-frame's window is the contiguous run
// of rows [win, win + n_valid) with win = (slot - n_valid + 1) mod cap.
// One thread per (state, angle); every counter then advances by one. One CTA.
__global__ void __launch_bounds__(256) step_begin_kernel(long long* ctr, FrameState* fs, int W,
                                                         int n_pairs, const double* inv_freq,
                                                         int n_sub, int B, int sub_cap,
                                                         int sub_mirror) {
  __shared__ long long t0[kMaxStreams];
  griddep_wait();
  griddep_launch();
  for (int b = threadIdx.x; b < B; b += blockDim.x) t0[b] = ctr[b];
  __syncthreads();
  const int per = 1 + n_sub;
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = threadIdx.x; i < B * per * n_pairs; i += blockDim.x) {
    const int st = i / n_pairs, m = i - st * n_pairs;
    const int b = st / per, k = st - b * per;
    const long long t = k == 0 ? t0[b] : t0[b] * n_sub + (k - 1);
    const int wnd = k == 0 ? W + 1 : n_sub * (W + 1);
    const int cap = k == 0 ? W + 1 : sub_cap;
    FrameState* f = fs + st;
    if (m == 0) {
      const int slot = int(t % cap);
      const int nv = int(t < wnd - 1 ? t : wnd - 1) + 1;
      f->t = t;
      f->slot = slot;
      f->n_valid = nv;
      f->win = (k > 0 && sub_mirror) ? (slot - nv + 1 + cap) % cap : 0;
    }
    double sn, cs;
    sincos(fmod(double(t) * inv_freq[m], two_pi), &sn, &cs);
    f->rope_t[m] = make_float2(float(cs), float(sn));
  }
  __syncthreads();
  for (int b = threadIdx.x; b < B; b += blockDim.x) ctr[b] = t0[b] + 1;
}

// ---------------------------------------------------------------- self-test
// Exercises the bounded-wait path every tcgen05 kernel relies on: an mbarrier
// that nobody arrives on is waited for with the same helper and a short
// limit; the wait must give up and record FD_ERR_TIMEOUT in *status.
__global__ void wait_timeout_selftest_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
}

// ---------------------------------------------------------------- embed
struct EmbedParams {
  const void* latent;     // [B][C'][H'][W'] io type
  int latent_bf16;
  int C, Hl, Wl, p;       // latent channels, rows, columns, patch
  int tok_w, L;           // L tokens per frame of one stream
  int M;                  // B L rows
  int c_in;               // C' p^2
  const float* wT;        // [c_in][D] (transposed projection)
  const float* b;         // [D]
  int D;
  float* x32;             // [M][D]
  void* xb;               // [M][D] storage type
  float* ssq;             // [M][D/32]
  int* status;            // device status word (bounds-checked build)
};

constexpr int kEmbedTok = 16;          // tokens per CTA
constexpr int kEmbedThreads = 256;     // each thread: 4 consecutive columns of every token

// One CTA = kEmbedTok tokens x all D columns (D a multiple of 32). The
// gathered latent values of the CTA's tokens sit in shared memory, channel-
// major so that one 16-byte broadcast read serves four tokens;
// thread i accumulates columns 4i .. 4i+3 of every token in registers, reading
// one 16-byte row of the transposed projection per input channel, so each
// weight load feeds kEmbedTok x 4 FMAs and every store of x (fp32 and storage
// type) is a contiguous run across the warp. The sum of squares of each
// 32-column chunk comes from the 8 lanes that own it.
template <typename T>
__global__ void __launch_bounds__(kEmbedThreads) embed_kernel(EmbedParams p) {
  extern __shared__ float u[];                          // [c_in][kEmbedTok]
  griddep_wait();
  griddep_launch();
  const int n0 = blockIdx.x * kEmbedTok;
  for (int idx = threadIdx.x; idx < kEmbedTok * p.c_in; idx += blockDim.x) {
    const int tk = idx / p.c_in, ch = idx - tk * p.c_in;
    const int n = n0 + tk;
    float v = 0.f;
    if (n < p.M) {
      const int b = n / p.L, nt = n - b * p.L;             // stream, token
      const int c = ch / (p.p * p.p), dy = (ch / p.p) % p.p, dx = ch % p.p;
      const int i = nt / p.tok_w, j = nt - (nt / p.tok_w) * p.tok_w;
      const size_t off = ((size_t(b) * p.C + c) * p.Hl + i * p.p + dy) * p.Wl + j * p.p + dx;
      if (FD_IN_BOUNDS(i * p.p + dy < p.Hl && j * p.p + dx < p.Wl, p.status))
        v = p.latent_bf16 ? __bfloat162float(static_cast<const bf16*>(p.latent)[off])
                          : static_cast<const float*>(p.latent)[off];
    }
    u[ch * kEmbedTok + tk] = v;
  }
  __syncthreads();
  const int parts = p.D / 32, lane = threadIdx.x & 31;
  // column groups of 4 kEmbedThreads; a lane past D computes on column 0 and
  // stores nothing, so every lane takes part in the shuffles
  for (int c0 = 0; c0 < p.D; c0 += 4 * kEmbedThreads) {
    const int col = c0 + 4 * threadIdx.x;
    if (c0 + 4 * (threadIdx.x & ~31) >= p.D) break;      // whole warp past D
    const bool active = col < p.D;
    const int cc = active ? col : 0;
    const float4 bd = __ldg(reinterpret_cast<const float4*>(p.b + cc));
    float4 acc[kEmbedTok];
#pragma unroll
    for (int t = 0; t < kEmbedTok; ++t) acc[t] = bd;
    const float4* w = reinterpret_cast<const float4*>(p.wT + cc);
    const int wstride = p.D / 4;
#pragma unroll 4
    for (int ch = 0; ch < p.c_in; ++ch) {
      const float4 wv = __ldg(w + size_t(ch) * wstride);
      const float4* uc = reinterpret_cast<const float4*>(u + ch * kEmbedTok);   // broadcast
#pragma unroll
      for (int t4 = 0; t4 < kEmbedTok / 4; ++t4) {
        const float4 a4 = uc[t4];
        const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int t = 4 * t4 + k;
          acc[t].x = fmaf(a[k], wv.x, acc[t].x);
          acc[t].y = fmaf(a[k], wv.y, acc[t].y);
          acc[t].z = fmaf(a[k], wv.z, acc[t].z);
          acc[t].w = fmaf(a[k], wv.w, acc[t].w);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kEmbedTok; ++t) {
      const int n = n0 + t;
      const float4 o = acc[t];
      float s = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (active && n < p.M) {
        *reinterpret_cast<float4*>(p.x32 + size_t(n) * p.D + col) = o;
        const float v[4] = {o.x, o.y, o.z, o.w};
        store_quad<T>(static_cast<T*>(p.xb) + size_t(n) * p.D + col, v);
        if ((lane & 7) == 0) p.ssq[size_t(n) * parts + col / 32] = s;
      }
    }
  }
}

// ---------------------------------------------------------------- MLP input (FP8)
// FP8 MLP (paper Sec. 4.6, static-calibrated FP8 quantization of the MLP
// layers): the first MLP Linear multiplies the FP8 image of its own input,
// the RMSNorm output a = x r g (r = 1/sqrt(mean(x^2) + eps), gain g), with
// the static scale s_a: x8 = e4m3(a / s_a), round to nearest even,
// saturating. With amax set (calibration of the unquantized path) the kernel
// records max |a| instead and writes nothing. r comes from the per-32-column
// sums of squares the producer of x emitted. One warp per row; D a multiple
// of 128. Bound by memory (x read once, one byte written per element).
struct NormQuantParams {
  const float* x32;       // [M][D] residual stream
  const float* ssq;       // [M][D/32] sums of squares of x32
  const float* g;         // [D] RMSNorm gain
  uint8_t* x8;            // [M][D] E4M3 codes of a / s_a (null with amax)
  unsigned* amax;         // calibration: max |a| as float bits (null: quantize)
  int M, D;
  float inv_d, eps;
  float q_inv;            // 1 / s_a
};

__global__ void __launch_bounds__(256) mlp_norm_quant_kernel(NormQuantParams p) {
  griddep_wait();
  griddep_launch();
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= p.M) return;
  const int parts = p.D / 32;
  float s = 0.f;
  for (int i = lane; i < parts; i += 32) s += p.ssq[size_t(row) * parts + i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float r = rsqrtf(s * p.inv_d + p.eps);
  const float4* x = reinterpret_cast<const float4*>(p.x32 + size_t(row) * p.D);
  const float4* g = reinterpret_cast<const float4*>(p.g);
  float m = 0.f;
  for (int c = lane; c < p.D / 4; c += 32) {
    const float4 v = x[c], gg = __ldg(g + c);
    const float a0 = v.x * r * gg.x, a1 = v.y * r * gg.y, a2 = v.z * r * gg.z, a3 = v.w * r * gg.w;
    if (p.amax) {
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a0), fabsf(a1)), fmaxf(fabsf(a2), fabsf(a3))));
    } else {
      const __nv_fp8x2_storage_t lo =
          __nv_cvt_float2_to_fp8x2(make_float2(a0 * p.q_inv, a1 * p.q_inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi =
          __nv_cvt_float2_to_fp8x2(make_float2(a2 * p.q_inv, a3 * p.q_inv), __NV_SATFINITE, __NV_E4M3);
      reinterpret_cast<uint32_t*>(p.x8 + size_t(row) * p.D)[c] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
  }
  if (p.amax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) atomicMax(p.amax, __float_as_uint(m));   // non-negative floats order as their bits
  }
}

// ---------------------------------------------------------------- simt_gemm
// C[M][N] = A[M][K] * B[N][K]^T, fp32, one thread per row and 64 columns,
// then the fused epilogue. CTA = 128 rows x 64 columns; K in chunks of 32.
template <int KIND, int DH>
__global__ void __launch_bounds__(128) simt_gemm_kernel(const float* A, const float* B, int K,
                                                        EpiParams p) {
  __shared__ float Bs[64][33];
  griddep_wait();
  griddep_launch();
  const int row = blockIdx.x * 128 + threadIdx.x;
  const int col0 = blockIdx.y * 64;
  float acc[64];
#pragma unroll
  for (int c = 0; c < 64; ++c) acc[c] = 0.f;
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int idx = threadIdx.x; idx < 64 * 32; idx += 128) {
      const int c = idx / 32, kk = idx % 32;
      Bs[c][kk] = B[size_t(col0 + c) * K + k0 + kk];
    }
    __syncthreads();
    if (row < p.M) {
      const float* a = A + size_t(row) * K + k0;
      for (int kk = 0; kk < 32; ++kk) {
        const float av = a[kk];
#pragma unroll
        for (int c = 0; c < 64; ++c) acc[c] = fmaf(av, Bs[c][kk], acc[c]);
      }
    }
    __syncthreads();
  }
  if (row < p.M) {
    const float rs = (epi_normed(KIND) && p.ssq) ? row_scale(p, row) : 1.f;
    epilogue64<KIND, float, DH>(p, row, col0, acc, rs);
  }
}

// ---------------------------------------------------------------- simt_attn
struct AttnParams {
  const void* q;          // [H][B][L][Dh]
  const void* kc;         // [B][G][kv_rows][Dh]
  const void* vtc;        // [B][G][Dh][vt_pitch]
  void* o;                // [B][L][H*Dh]
  int L, H, G, kv_rows, vt_pitch;
  int B, fs_stride;       // streams; FrameStates per stream
  float scale_log2;       // log2(e) / sqrt(Dh)
  const FrameState* fs;
  int* status;
};

// One thread per query row, keys in tiles of 32 staged in shared memory,
// online softmax in base 2. Keys [0, n_valid*L) are the valid ring slots.
template <int DH>
__global__ void __launch_bounds__(64) simt_attn_kernel(AttnParams p) {
  griddep_wait();
  griddep_launch();
  __shared__ float Ks[32][DH + 1];
  __shared__ float Vs[32][DH + 1];
  const int h = blockIdx.y, g = h / (p.H / p.G), bs = blockIdx.z;
  const int row = blockIdx.x * 64 + threadIdx.x;
  int n_keys = p.fs[size_t(bs) * p.fs_stride].n_valid * p.L;
  if (!FD_IN_BOUNDS(n_keys <= p.kv_rows, p.status)) n_keys = 0;
  const float* qp = static_cast<const float*>(p.q) +
                    ((size_t(h) * p.B + bs) * p.L + (row < p.L ? row : 0)) * DH;
  float q[DH], o[DH];
#pragma unroll
  for (int d = 0; d < DH; ++d) { q[d] = qp[d] * p.scale_log2; o[d] = 0.f; }
  float m = -INFINITY, l = 0.f;
  const float* kg = static_cast<const float*>(p.kc) + (size_t(bs) * p.G + g) * p.kv_rows * DH;
  const float* vg = static_cast<const float*>(p.vtc) + (size_t(bs) * p.G + g) * DH * p.vt_pitch;
  for (int k0 = 0; k0 < n_keys; k0 += 32) {
    for (int idx = threadIdx.x; idx < 32 * DH; idx += 64) {
      const int j = idx / DH, d = idx % DH;
      const bool ok = k0 + j < n_keys;
      Ks[j][d] = ok ? kg[size_t(k0 + j) * DH + d] : 0.f;
      const int jj = idx % 32, dd = idx / 32;          // transposed read of V
      Vs[jj][dd] = (k0 + jj < n_keys) ? vg[size_t(dd) * p.vt_pitch + k0 + jj] : 0.f;
    }
    __syncthreads();
    const int nk = min(32, n_keys - k0);
    float s[32];
    float mt = m;
    for (int j = 0; j < 32; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int d = 0; d < DH; ++d) acc = fmaf(q[d], Ks[j][d], acc);
      s[j] = j < nk ? acc : -INFINITY;
      mt = fmaxf(mt, s[j]);
    }
    const float corr = exp2f(m - mt);
    l *= corr;
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] *= corr;
    for (int j = 0; j < 32; ++j) {
      const float pj = exp2f(s[j] - mt);
      l += pj;
#pragma unroll
      for (int d = 0; d < DH; ++d) o[d] = fmaf(pj, Vs[j][d], o[d]);
    }
    m = mt;
    __syncthreads();
  }
  if (row < p.L) {
    const float inv = 1.f / l;
    float* op = static_cast<float*>(p.o) + (size_t(bs) * p.L + row) * p.H * DH + size_t(h) * DH;
#pragma unroll
    for (int d = 0; d < DH; ++d) op[d] = o[d] * inv;
  }
}

}  // namespace fd
