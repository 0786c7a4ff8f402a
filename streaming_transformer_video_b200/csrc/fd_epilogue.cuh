// fd_epilogue.cuh — fused GEMM epilogues of the FlashDecoder step.
//
// A GEMM thread owns one token row and 64 consecutive accumulator columns
// (fp32). The epilogue finishes the layer's math on them in registers and
// writes the result where the next kernel wants it:
//   QKV    RMSNorm row scale + bias, KV-norm, 3D-RoPE, Q to its buffer and
//          K/V into the frame's ring slot            (paper Sec. 3.2, 3.3, Eq. 2)
//   RESID  residual add into the fp32 stream x, its storage-type copy and
//          the per-32-column sums of squares the next RMSNorm needs
//   GELU   RMSNorm row scale + bias + exact GELU -> MLP hidden
//   FINAL  [RMSNorm row scale] + bias -> unpatchify scatter into NCTHW pixels
//          (Sec. 3.4, Step 3: depth-to-space)
//   UP     bias -> temporal upsampling (Sec. 3.4, Eq. 3): output channels
//          [tau D, (tau+1) D) become the residual stream of sub-frame tau
//          (fp32 copy, storage-type copy, per-32-column sums of squares)
// FP8 MLP (Sec. 4.6, static per-tensor scales; the MLP-up's FP8 input
// e4m3(RMSNorm(x) / s_a) is written by mlp_norm_quant_kernel in between):
//   RESID_Q  as RESID, without the storage-type copy of x (the MLP-up reads
//            the FP8 input instead)
//   GELU_Q   dequantize (acc s_a s_w1) + bias + GELU -> FP8 hidden h / s_h
//            (the MLP-down's A operand)
//   RESID with acc_scale = s_h s_w2 dequantizes the MLP-down product
// Calibration (unquantized path): RESID and GELU can record max |value| of
// their outputs into a device word (float bits, atomicMax).
//
// RMSNorm fusion: the gain g is folded into the following weight matrix at
// create time, so RMSNorm(x) W^T = diag(r) (x (W diag g)^T) with
// r = 1/sqrt(mean(x^2) + eps). The producer of x emits sums of x^2 over each
// 32-column chunk; the consumer adds them up per row (deterministic order).
#pragma once

#include "fd_common.cuh"

namespace fd {

enum EpiKind {
  EPI_QKV = 0, EPI_RESID = 1, EPI_GELU = 2, EPI_FINAL = 3, EPI_UP = 4,
  EPI_RESID_Q = 5, EPI_GELU_Q = 6
};

// Kinds whose A operand is an RMSNorm input (their rows get the row scale);
// a null EpiParams::ssq turns the scale off (the spatial MLP's second layer).
constexpr bool epi_normed(int kind) {
  return kind == EPI_QKV || kind == EPI_GELU || kind == EPI_FINAL;
}

struct EpiParams {
  int M;                 // rows: n_sub sub-frames x B video streams x L tokens,
                         // row = (tau B + b) L + n (n_sub = 1: row = b L + n)
  int L;                 // tokens per frame of one stream
  int B;                 // video streams
  int N;                 // GEMM output columns
  const float* bias;     // [N]
  // RMSNorm row scale (QKV, GELU, FINAL; none when ssq is null)
  const float* ssq;      // [M][ssq_parts] sums of squares of x
  int ssq_parts;
  float inv_d;           // 1 / D
  float eps;
  // RESID (UP: the same three buffers with a leading sub-frame index)
  float* x32;            // [M][D] fp32 residual stream (updated in place)
  void* xb;              // [M][D] storage-type copy (next GEMM's A operand)
  float* ssq_out;        // [M][D/32]
  int D;
  // QKV
  void* q;               // [H][M][Dh]
  void* kc;              // this block's keys   [B][G][kv_rows][Dh]
  void* vtc;             // this block's values [B][G][Dh][vt_pitch] (transposed)
  int H, G, Dh;
  int kv_rows;           // rows of one (stream, group) slab of the ring
  int vt_pitch;          // row pitch of the transposed values (elements)
  int kv_mirror;         // mirrored ring: rows between a key's two copies (0: one copy)
  const float* gk;       // [Dh] KV-norm gains
  const float* gv;
  int kv_norm;
  const FrameState* fs;  // state of stream b, sub-frame tau: fs[b * fs_stride + tau]
  int fs_stride;
  const float2* rope_row;  // [tok_h][d_s/2] (cos, sin)
  const float2* rope_col;  // [tok_w][d_s/2]
  int tok_w;
  // GELU
  void* hout;            // [M][N]
  // FINAL
  void* out;             // [B][C][r_t][tok_h*P][tok_w*P]
  size_t out_stride;     // pixels per stream
  int out_bf16;          // pixel element type
  int P;                 // pixels per token side
  int tok_h;
  int pl_mul, pl_add;    // column block c = col / P^2 of sub-frame tau's row goes
                         // to pixel frame c * pl_mul + pl_add + tau of the
                         // [C * r_t] output frames
  // FP8 MLP
  float acc_scale;       // dequantization of the accumulator (1: none)
  float q_inv;           // 1 / static scale of the FP8 output
  // calibration: max |output| as float bits (null: off)
  unsigned* amax;
  // bounds of the bounds-checked build (FD_IN_BOUNDS)
  int* status;           // device status word
  int n_sub;             // UP: sub-frames r_t of x32 / xb / ssq_out
  int out_frames;        // FINAL: pixel frames per stream (C r_t)
};

// 64 floats * q_inv -> 64 E4M3 bytes (round to nearest even, saturating at
// +-448), as four 16-byte stores.
__device__ __forceinline__ void store_e4m3_64(uint8_t* dst, const float* v, float q_inv) {
#pragma unroll
  for (int c = 0; c < 64; c += 16) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
          make_float2(v[c + 4 * i] * q_inv, v[c + 4 * i + 1] * q_inv), __NV_SATFINITE, __NV_E4M3);
      const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
          make_float2(v[c + 4 * i + 2] * q_inv, v[c + 4 * i + 3] * q_inv), __NV_SATFINITE, __NV_E4M3);
      w[i] = uint32_t(lo) | (uint32_t(hi) << 16);
    }
    *reinterpret_cast<uint4*>(dst + c) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Four consecutive biases with one 16-byte load (every bias slice an
// epilogue reads starts on a 32-column boundary of a 256-byte aligned array).
__device__ __forceinline__ float4 bias4(const float* b, int col) {
  return __ldg(reinterpret_cast<const float4*>(b + col));
}

// v[c] = v[c] * s + b[col + c], c < n (n a multiple of 4)
template <int n>
__device__ __forceinline__ void scale_bias(float* v, float s, const float* b, int col) {
#pragma unroll
  for (int c = 0; c < n; c += 4) {
    const float4 bb = bias4(b, col + c);
    v[c] = v[c] * s + bb.x;
    v[c + 1] = v[c + 1] * s + bb.y;
    v[c + 2] = v[c + 2] * s + bb.z;
    v[c + 3] = v[c + 3] * s + bb.w;
  }
}

__device__ __forceinline__ void record_amax(unsigned* amax, const float* v) {
  float m = 0.f;
#pragma unroll
  for (int c = 0; c < 64; ++c) m = fmaxf(m, fabsf(v[c]));
  atomicMax(amax, __float_as_uint(m));     // non-negative floats order as their bits
}

__device__ __forceinline__ float row_scale(const EpiParams& p, int row) {
  // ssq_parts = D / 32 is even (D is a multiple of 64): independent loads in
  // flight, four partial sums
  const float2* s = reinterpret_cast<const float2*>(p.ssq + size_t(row) * p.ssq_parts);
  const int n2 = p.ssq_parts / 2;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int i = 0;
#pragma unroll 4
  for (; i + 2 <= n2; i += 2) {
    const float2 u = s[i], v = s[i + 1];
    a0 += u.x; a1 += u.y; a2 += v.x; a3 += v.y;
  }
  if (i < n2) { const float2 u = s[i]; a0 += u.x; a1 += u.y; }
  return rsqrtf(((a0 + a1) + (a2 + a3)) * p.inv_d + p.eps);
}

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

// In-place 3D-RoPE of one head vector v[DH] of token n of a frame with state
// fs: pairs (2m, 2m+1) of the temporal part [0, DH/4) rotate by the frame's
// angle, the row part [DH/4, DH/4 + 3DH/8) by the token's grid row, the
// column part by its column.
template <int DH>
__device__ __forceinline__ void rope_head(float* v, int n, const FrameState* fs,
                                          const EpiParams& p) {
  constexpr int dt = DH / 4, ds = 3 * DH / 8;
  const int i = n / p.tok_w, j = n - (n / p.tok_w) * p.tok_w;
  const float2* rr = p.rope_row + size_t(i) * (ds / 2);
  const float2* rc = p.rope_col + size_t(j) * (ds / 2);
#pragma unroll
  for (int m = 0; m < dt / 2; ++m) {
    const float2 cs = fs->rope_t[m];
    const float a = v[2 * m], b = v[2 * m + 1];
    v[2 * m] = a * cs.x - b * cs.y;
    v[2 * m + 1] = a * cs.y + b * cs.x;
  }
#pragma unroll
  for (int m = 0; m < ds / 2; ++m) {
    const float2 cs = __ldg(rr + m);
    float* w = v + dt + 2 * m;
    const float a = w[0], b = w[1];
    w[0] = a * cs.x - b * cs.y;
    w[1] = a * cs.y + b * cs.x;
  }
#pragma unroll
  for (int m = 0; m < ds / 2; ++m) {
    const float2 cs = __ldg(rc + m);
    float* w = v + dt + ds + 2 * m;
    const float a = w[0], b = w[1];
    w[0] = a * cs.x - b * cs.y;
    w[1] = a * cs.y + b * cs.x;
  }
}

template <int DH>
__device__ __forceinline__ void rms_head(float* v, const float* g, float eps) {
  float s = 0.f;
#pragma unroll
  for (int d = 0; d < DH; ++d) s += v[d] * v[d];
  const float r = rsqrtf(s * (1.f / DH) + eps);
#pragma unroll
  for (int d = 0; d < DH; ++d) v[d] = v[d] * r * __ldg(g + d);
}

// Unpatchify / PixelShuffle scatter of 64 finished columns of token `row`:
// 64 / P output rows of P pixels each; column (b*P + dy)*P + dx maps to pixel
// frame b*pl_mul + pl_add + tau, pixel row i*P+dy, pixels j*P .. j*P+P-1,
// where tau is the sub-frame of the row (0 unless the launch covers several).
// The linear head has b = c*r_t + tau (pl_mul 1, pl_add 0); the spatial MLP
// has b = c (pl_mul r_t; pl_add tau when each sub-frame is its own launch).
// P is a template parameter so the accumulator stays in registers.
template <int P>
__device__ __forceinline__ void pixel_scatter(const EpiParams& p, int row, int col0,
                                              const float* acc) {
  const int bq = row / p.L, n = row - bq * p.L;            // (sub-frame, stream), token
  const int b = bq % p.B, tau = bq / p.B;
  const int i = n / p.tok_w, j = n - (n / p.tok_w) * p.tok_w;
  const size_t out_w = size_t(p.tok_w) * P;
  const size_t plane = size_t(p.tok_h) * P * out_w;      // one [H][W] pixel frame
#pragma unroll
  for (int s = 0; s < 64; s += P) {
    const int col = col0 + s;
    const int ct = (col / (P * P)) * p.pl_mul + p.pl_add + tau;
    const int dy = (col / P) % P;
    const size_t off = size_t(b) * p.out_stride + size_t(ct) * plane +
                       (size_t(i) * P + dy) * out_w + size_t(j) * P;
    if (!FD_IN_BOUNDS(ct < p.out_frames && i < p.tok_h && off + P <= size_t(b + 1) * p.out_stride,
                      p.status))
      continue;
    if (p.out_bf16) store_vec<bf16, P>(static_cast<bf16*>(p.out) + off, acc + s);
    else store_vec<float, P>(static_cast<float*>(p.out) + off, acc + s);
  }
}

// Residual epilogue (RESID, RESID_Q) for a whole warp: thread `lane` holds
// columns col0 .. col0+63 of row row0 + lane. Done row by row, each thread
// would touch its own 256-byte row of x, so every warp-wide access would span
// 32 rows. Instead the accumulator goes through a [32][kResidPitch] fp32 tile
// of shared memory, 32 columns at a time, and 8 lanes cover one row: every
// load and store of x (fp32), its storage-type copy and the sums of squares
// is then a run of 128 (or 64) contiguous bytes per row. Rows past M are
// skipped; the warp stays converged for the shuffles.
constexpr int kResidPitch = 36;          // floats per tile row (conflict-free float4)

template <int KIND, typename T>
__device__ __forceinline__ void resid_epilogue64(const EpiParams& p, int row0, int col0,
                                                 const float* acc, float* tile, int lane) {
  const int parts = p.D / 32;
  const float sc = p.acc_scale;
  const int c4 = lane & 7, sub = lane >> 3;
  // all 16 of this lane's residual reads first (they do not depend on the
  // accumulator), so that they are in flight together
  float4 xin[2][8];
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int row = row0 + 4 * it + sub;
      xin[h][it] = row < p.M ? *reinterpret_cast<const float4*>(p.x32 + size_t(row) * p.D + col0 +
                                                               32 * h + 4 * c4)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float4* mine = reinterpret_cast<float4*>(tile + lane * kResidPitch);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      mine[k] = make_float4(acc[32 * h + 4 * k], acc[32 * h + 4 * k + 1], acc[32 * h + 4 * k + 2],
                            acc[32 * h + 4 * k + 3]);
    __syncwarp();
    const int col = col0 + 32 * h + 4 * c4;
    const float4 bb = bias4(p.bias, col);
    float m = 0.f;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int rr = 4 * it + sub, row = row0 + rr;
      const bool in = row < p.M;
      const float4 a = reinterpret_cast<const float4*>(tile + rr * kResidPitch)[c4];
      float4 o = xin[h][it];
      o.x += a.x * sc + bb.x;
      o.y += a.y * sc + bb.y;
      o.z += a.z * sc + bb.z;
      o.w += a.w * sc + bb.w;
      if (in) {
        *reinterpret_cast<float4*>(p.x32 + size_t(row) * p.D + col) = o;
        if constexpr (KIND == EPI_RESID) {
          const float v[4] = {o.x, o.y, o.z, o.w};
          store_quad<T>(static_cast<T*>(p.xb) + size_t(row) * p.D + col, v);
        }
        m = fmaxf(m, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
      }
      float ss = o.x * o.x + o.y * o.y + o.z * o.z + o.w * o.w;
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      if (in && c4 == 0) p.ssq_out[size_t(row) * parts + (col0 + 32 * h) / 32] = ss;
    }
    if (p.amax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) atomicMax(p.amax, __float_as_uint(m));
    }
    __syncwarp();
  }
}

// QKV epilogue for a whole warp (tcgen05 path, bf16, D_h = 64): thread `lane`
// holds head col0 / 64 of token row0 + lane. The math is the per-thread QKV
// epilogue's; the query and key rows (128 bytes per token) then go through a
// [32][kQkvPitch] bf16 tile of shared memory so that 8 lanes store one token's
// row: each warp-wide store covers 4 whole rows instead of touching 32. The
// transposed value rows keep the per-thread stores (32 consecutive keys of
// one dimension per warp-wide store are already contiguous). Rows past M do
// the arithmetic on clamped indices and store nothing.
constexpr int kQkvPitch = 72;            // bf16 per tile row (conflict-free 16-byte access)

__device__ __forceinline__ void warp_store_rows64(bf16* dst, const float* v, bf16* tile, int lane) {
  // this lane's row -> tile, then 4 rows per step, 16 bytes per lane
  uint4* mine = reinterpret_cast<uint4*>(tile + lane * kQkvPitch);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 b2 = __floats2bfloat162_rn(v[8 * k + 2 * i], v[8 * k + 2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b2);
    }
    mine[k] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncwarp();
  const int c = lane & 7, sub = lane >> 3;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int rr = 4 * it + sub;
    bf16* d = reinterpret_cast<bf16*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(dst), rr));
    const uint4 u = reinterpret_cast<const uint4*>(tile + rr * kQkvPitch)[c];
    if (d) reinterpret_cast<uint4*>(d)[c] = u;
  }
  __syncwarp();
}

__device__ __forceinline__ void qkv_epilogue64(const EpiParams& p, int row, int col0, float* acc,
                                               float rs, bf16* tile, int lane) {
  constexpr int DH = 64;
  const bool valid = row < p.M;
  const int rowc = valid ? row : 0;
  const int bq = rowc / p.L, n = rowc - bq * p.L;          // (sub-frame, stream), token
  const int b = bq % p.B, tau = bq / p.B;
  const FrameState* fs = p.fs + size_t(b) * p.fs_stride + tau;
  float* v = acc;
  const int head = col0 / DH;
  scale_bias<DH>(v, rs, p.bias, col0);
  bf16* dst = nullptr;
  if (head < p.H) {                                        // query head (warp-uniform)
    rope_head<DH>(v, n, fs, p);
    if (valid) dst = static_cast<bf16*>(p.q) + (size_t(head) * p.M + row) * DH;
    warp_store_rows64(dst, v, tile, lane);
  } else if (head < p.H + p.G) {                           // key group
    const int g = head - p.H;
    if (p.kv_norm) rms_head<DH>(v, p.gk, p.eps);
    rope_head<DH>(v, n, fs, p);
    const int key = fs->slot * p.L + n;
    if (valid && FD_IN_BOUNDS(fs->slot >= 0 && key + p.kv_mirror < p.kv_rows && bq * p.L < p.M,
                              p.status))
      dst = static_cast<bf16*>(p.kc) + ((size_t(b) * p.G + g) * p.kv_rows + key) * DH;
    warp_store_rows64(dst, v, tile, lane);
    if (p.kv_mirror)                                       // uniform: the second copy
      warp_store_rows64(dst ? dst + size_t(p.kv_mirror) * DH : nullptr, v, tile, lane);
  } else {                                                 // value group
    const int g = head - p.H - p.G;
    if (p.kv_norm) rms_head<DH>(v, p.gv, p.eps);
    const int key = fs->slot * p.L + n;
    if (valid && FD_IN_BOUNDS(fs->slot >= 0 && key + p.kv_mirror < p.kv_rows &&
                              key + p.kv_mirror < p.vt_pitch && g < p.G && bq * p.L < p.M,
                              p.status)) {
      bf16* d = static_cast<bf16*>(p.vtc) + (size_t(b) * p.G + g) * DH * p.vt_pitch + key;
#pragma unroll
      for (int i = 0; i < DH; ++i) d[size_t(i) * p.vt_pitch] = __float2bfloat16_rn(v[i]);
      if (p.kv_mirror) {
#pragma unroll
        for (int i = 0; i < DH; ++i)
          d[size_t(i) * p.vt_pitch + p.kv_mirror] = __float2bfloat16_rn(v[i]);
      }
    }
  }
}

// acc[64]: columns col0 .. col0+63 of token `row` (row < M guaranteed).
template <int KIND, typename T, int DH>
__device__ __forceinline__ void epilogue64(const EpiParams& p, int row, int col0, float* acc,
                                           float rs) {
  if constexpr (KIND == EPI_QKV) {
    const int bq = row / p.L, n = row - bq * p.L;          // (sub-frame, stream), token
    const int b = bq % p.B, tau = bq / p.B;
    const FrameState* fs = p.fs + size_t(b) * p.fs_stride + tau;
#pragma unroll
    for (int hh = 0; hh < 64 / DH; ++hh) {
      float* v = acc + hh * DH;
      const int col = col0 + hh * DH;
      const int head = col / DH;
      scale_bias<DH>(v, rs, p.bias, col);
      if (head < p.H) {                                   // query head
        rope_head<DH>(v, n, fs, p);
        T* dst = static_cast<T*>(p.q) + (size_t(head) * p.M + row) * DH;
        store_vec<T, DH>(dst, v);
      } else if (head < p.H + p.G) {                      // key group
        const int g = head - p.H;
        if (p.kv_norm) rms_head<DH>(v, p.gk, p.eps);
        rope_head<DH>(v, n, fs, p);
        const int key = fs->slot * p.L + n;
        if (!FD_IN_BOUNDS(fs->slot >= 0 && key + p.kv_mirror < p.kv_rows && bq * p.L < p.M,
                          p.status))
          continue;
        T* dst = static_cast<T*>(p.kc) + ((size_t(b) * p.G + g) * p.kv_rows + key) * DH;
        store_vec<T, DH>(dst, v);
        if (p.kv_mirror) store_vec<T, DH>(dst + size_t(p.kv_mirror) * DH, v);
      } else {                                            // value group
        const int g = head - p.H - p.G;
        if (p.kv_norm) rms_head<DH>(v, p.gv, p.eps);
        const int key = fs->slot * p.L + n;
        if (!FD_IN_BOUNDS(fs->slot >= 0 && key + p.kv_mirror < p.kv_rows &&
                          key + p.kv_mirror < p.vt_pitch && g < p.G && bq * p.L < p.M, p.status))
          continue;
        T* dst = static_cast<T*>(p.vtc) + (size_t(b) * p.G + g) * DH * p.vt_pitch + key;
#pragma unroll
        for (int d = 0; d < DH; ++d) dst[size_t(d) * p.vt_pitch] = from_f<T>(v[d]);
        if (p.kv_mirror) {
#pragma unroll
          for (int d = 0; d < DH; ++d) dst[size_t(d) * p.vt_pitch + p.kv_mirror] = from_f<T>(v[d]);
        }
      }
    }
  } else if constexpr (KIND == EPI_RESID || KIND == EPI_RESID_Q) {
    float* x = p.x32 + size_t(row) * p.D + col0;
    const float sc = p.acc_scale;
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
      float4 o = *reinterpret_cast<const float4*>(x + c);
      const float4 bb = bias4(p.bias, col0 + c);
      o.x += acc[c + 0] * sc + bb.x;
      o.y += acc[c + 1] * sc + bb.y;
      o.z += acc[c + 2] * sc + bb.z;
      o.w += acc[c + 3] * sc + bb.w;
      *reinterpret_cast<float4*>(x + c) = o;
      acc[c + 0] = o.x; acc[c + 1] = o.y; acc[c + 2] = o.z; acc[c + 3] = o.w;
    }
    if constexpr (KIND == EPI_RESID)
      store_vec<T, 64>(static_cast<T*>(p.xb) + size_t(row) * p.D + col0, acc);
    if (p.amax) record_amax(p.amax, acc);
    const int parts = p.D / 32;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) s += acc[h * 32 + c] * acc[h * 32 + c];
      p.ssq_out[size_t(row) * parts + col0 / 32 + h] = s;
    }
  } else if constexpr (KIND == EPI_GELU) {
    scale_bias<64>(acc, rs, p.bias, col0);
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = gelu_erf(acc[c]);
    store_vec<T, 64>(static_cast<T*>(p.hout) + size_t(row) * p.N + col0, acc);
    if (p.amax) record_amax(p.amax, acc);
  } else if constexpr (KIND == EPI_GELU_Q) {
    scale_bias<64>(acc, p.acc_scale, p.bias, col0);
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = gelu_erf(acc[c]);
    store_e4m3_64(static_cast<uint8_t*>(p.hout) + size_t(row) * p.N + col0, acc, p.q_inv);
  } else if constexpr (KIND == EPI_UP) {
    const int tau = col0 / p.D, c0 = col0 - tau * p.D;
    const size_t r = size_t(tau) * p.M + row;             // row of sub-frame tau
    if (!FD_IN_BOUNDS(tau < p.n_sub, p.status)) return;
    scale_bias<64>(acc, 1.f, p.bias, col0);
    float* x = p.x32 + r * p.D + c0;
#pragma unroll
    for (int c = 0; c < 64; c += 4)
      *reinterpret_cast<float4*>(x + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
    store_vec<T, 64>(static_cast<T*>(p.xb) + r * p.D + c0, acc);
    const int parts = p.D / 32;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < 32; ++c) s += acc[h * 32 + c] * acc[h * 32 + c];
      p.ssq_out[r * parts + c0 / 32 + h] = s;
    }
  } else {  // EPI_FINAL
    scale_bias<64>(acc, rs, p.bias, col0);
    if (p.P == 16) pixel_scatter<16>(p, row, col0, acc);
    else pixel_scatter<8>(p, row, col0, acc);
  }
}

}  // namespace fd
