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
// Frame state of one streamed frame with absolute index t in a ring of `cap`
// slots: slot = t mod cap; n_valid = min(t, cap - 1) + 1; temporal RoPE
// angles t * theta^(-2m/d_t) reduced mod 2 pi in fp64 so they stay exact for
// any stream length.
__device__ void frame_state(FrameState* fs, long long t, int cap, int head_dim, float theta) {
  fs->t = t;
  fs->slot = int(t % cap);
  fs->n_valid = int(t < cap - 1 ? t : cap - 1) + 1;
  const int dt = head_dim / 4;
  const double two_pi = 6.283185307179586476925286766559;
  for (int m = 0; m < dt / 2; ++m) {
    const double freq = pow(double(theta), -2.0 * m / dt);
    const double ang = fmod(double(t) * freq, two_pi);
    fs->rope_t[m] = make_float2(float(cos(ang)), float(sin(ang)));
  }
}

// B video streams, each with its own counter ctr[b] and 1 + n_sub states
// fs[b (1 + n_sub) + k]:
//   k = 0: latent frame t = ctr[b] in the backbone ring of W+1 frames;
//   k = 1 + tau, tau < n_sub (paper head, n_sub = r_t): sub-frame t r_t + tau
//   in the refinement ring of r_t (W+1) sub-frames (paper Sec. 3.4, Step 2).
// Every counter then advances by one. One CTA of 32 threads.
__global__ void step_begin_kernel(long long* ctr, FrameState* fs, int W, int head_dim,
                                  float theta, int n_sub, int B) {
  __shared__ long long t0[kMaxStreams];
  for (int b = threadIdx.x; b < B; b += blockDim.x) t0[b] = ctr[b];
  __syncthreads();
  const int per = 1 + n_sub;
  for (int i = threadIdx.x; i < B * per; i += blockDim.x) {
    const int b = i / per, k = i - b * per;
    if (k == 0) frame_state(fs + i, t0[b], W + 1, head_dim, theta);
    else frame_state(fs + i, t0[b] * n_sub + (k - 1), n_sub * (W + 1), head_dim, theta);
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
};

constexpr int kEmbedTok = 8;

// One CTA = kEmbedTok tokens; thread d handles columns d, d+256, ...
// Sums of squares per 32-column chunk come from a warp reduction (each warp
// owns whole 32-column chunks).
template <typename T>
__global__ void __launch_bounds__(256) embed_kernel(EmbedParams p) {
  extern __shared__ float u[];                          // [kEmbedTok][c_in]
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
      v = p.latent_bf16 ? __bfloat162float(static_cast<const bf16*>(p.latent)[off])
                        : static_cast<const float*>(p.latent)[off];
    }
    u[idx] = v;
  }
  __syncthreads();
  const int parts = p.D / 32;
  for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
    float acc[kEmbedTok];
    const float bd = __ldg(p.b + d);
#pragma unroll
    for (int t = 0; t < kEmbedTok; ++t) acc[t] = bd;
    for (int ch = 0; ch < p.c_in; ++ch) {
      const float w = __ldg(p.wT + size_t(ch) * p.D + d);
#pragma unroll
      for (int t = 0; t < kEmbedTok; ++t) acc[t] = fmaf(u[t * p.c_in + ch], w, acc[t]);
    }
#pragma unroll
    for (int t = 0; t < kEmbedTok; ++t) {
      const int n = n0 + t;
      float s = acc[t] * acc[t];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (n < p.M) {
        p.x32[size_t(n) * p.D + d] = acc[t];
        static_cast<T*>(p.xb)[size_t(n) * p.D + d] = from_f<T>(acc[t]);
        if ((threadIdx.x & 31) == 0) p.ssq[size_t(n) * parts + d / 32] = s;
      }
    }
  }
}

// ---------------------------------------------------------------- simt_gemm
// C[M][N] = A[M][K] * B[N][K]^T, fp32, one thread per row and 64 columns,
// then the fused epilogue. CTA = 128 rows x 64 columns; K in chunks of 32.
template <int KIND, int DH>
__global__ void __launch_bounds__(128) simt_gemm_kernel(const float* A, const float* B, int K,
                                                        EpiParams p) {
  __shared__ float Bs[64][33];
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
  __shared__ float Ks[32][DH + 1];
  __shared__ float Vs[32][DH + 1];
  const int h = blockIdx.y, g = h / (p.H / p.G), bs = blockIdx.z;
  const int row = blockIdx.x * 64 + threadIdx.x;
  const int n_keys = p.fs[size_t(bs) * p.fs_stride].n_valid * p.L;
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
