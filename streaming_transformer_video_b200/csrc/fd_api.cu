// fd_api.cu — host runtime and C ABI of the FlashDecoder streaming step.
//
// fd_create validates the configuration, packs the weights (RMSNorm gains
// folded into the following Linear, bf16 rounding), allocates the ring cache
// and every scratch buffer once, encodes the TMA tensor maps and builds one
// CUDA graph of the whole per-frame step (paper Sec. 4.6: the per-frame pass
// is a fixed, data-independent graph). fd_decode_frame replays that graph.
//
// Per-frame kernel sequence (bf16 configuration, all sm_100a):
//   step_begin -> embed -> n_blocks x [QKV GEMM (+norm, KV-norm, RoPE, ring
//   write) -> attention -> O-proj GEMM (+residual) -> MLP-up GEMM (+GELU) ->
//   MLP-down GEMM (+residual)] -> head
// Linear head: final GEMM (+norm, unpatchify).
// Paper head (Sec. 3.4): upsample GEMM (Eq. 3, one launch for all r_t
//   sub-frames) -> for each sub-frame tau in order: n_refine x [the five block
//   kernels on sub-frame tau, refinement ring] -> spatial GEMM (+norm, GELU)
//   -> final GEMM (PixelShuffle into pixel frame tau).
// The fp32 configuration runs the same sequence with CUDA-core kernels.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "fd_attn_tc.cuh"
#include "fd_gemm_tc.cuh"
#include "fd_simt.cuh"

using namespace fd;

namespace {

thread_local std::string g_last_error;

fd_status_t fail(fd_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

#define FD_CUDA(call)                                                                     \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess) {                                                              \
      cudaGetLastError();                                                                 \
      return fail(e_ == cudaErrorMemoryAllocation ? FD_ERR_OOM : FD_ERR_CUDA, "%s: %s", #call, \
                  cudaGetErrorString(e_));                                                \
    }                                                                                     \
  } while (0)

#define FD_TRY(expr)                     \
  do {                                   \
    fd_status_t s_ = (expr);             \
    if (s_ != FD_OK) return s_;          \
  } while (0)

// Consecutive kernels of the frame graph are linked by programmatic edges
// (programmatic dependent launch; every kernel orders its data accesses with
// griddep_wait). Builds with -DFD_PDL=0 use full dependencies instead.
#ifndef FD_PDL
#define FD_PDL 1
#endif
constexpr bool kUsePdl = FD_PDL != 0;

constexpr uint32_t kMagic = 0xFDEC0DE5u;
constexpr uint32_t kDead = 0xDEADFD00u;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

uint16_t f32_to_bf16_bits(float f) {        // round to nearest even
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return uint16_t((u >> 16) | ((u & 0xFFFF) ? 0x40 : 0));
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return uint16_t(u >> 16);
}

float bf16_bits_to_f32(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

fd_status_t get_encode() {
  if (g_encode) return FD_OK;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  FD_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q));
  if (q != cudaDriverEntryPointSuccess || !fn)
    return fail(FD_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return FD_OK;
}

// Tensor map (bf16 by default, or bytes for E4M3) with 128-byte swizzle.
// dims/strides innermost first; strides[i] is the byte pitch of dimension i+1.
fd_status_t make_tmap(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides, const uint32_t* box,
                      CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  FD_TRY(get_encode());
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(m, type, rank, const_cast<void*>(base),
                        reinterpret_cast<const cuuint64_t*>(dims),
                        reinterpret_cast<const cuuint64_t*>(strides),
                        reinterpret_cast<const cuuint32_t*>(box), estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FD_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FD_OK;
}

// Row-major [rows][cols] bf16 matrix read in boxes of box_rows x 64.
fd_status_t make_tmap_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols * 2};
  const uint32_t box[2] = {64, box_rows};
  return make_tmap(m, base, 2, dims, strides, box);
}

// Row-major [rows][cols] E4M3 matrix read in boxes of box_rows x 128 bytes.
fd_status_t make_tmap_2d_e4m3(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_rows) {
  const uint64_t dims[2] = {cols, rows};
  const uint64_t strides[1] = {cols};
  const uint32_t box[2] = {128, box_rows};
  return make_tmap(m, base, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

// FP8 E4M3 code of v: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits,
// no infinities; the largest finite value 448 = 1.75 * 2^8 is code 0x7E and
// 0x7F is NaN. Round to nearest, ties to even (the default rounding mode of
// nearbyint); magnitudes >= 448 after rounding saturate to 448.
uint8_t e4m3_encode(double v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(v);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int ex = 0;
  std::frexp(a, &ex);                       // a = m 2^ex, m in [0.5, 1)
  int e = std::max(ex - 1, -6);             // binade 2^e; subnormal spacing below 2^-6
  double q = std::nearbyint(std::ldexp(a, 3 - e));   // multiples of 2^(e-3)
  if (q >= 16.0) { q = 8.0; ++e; }          // rounded up into the next binade
  if (e == -6 && q < 8.0) return sign | uint8_t(q);               // subnormal (or zero)
  if (e > 8 || (e == 8 && q > 14.0)) return sign | 0x7E;          // beyond 448
  return sign | uint8_t(((e + 7) << 3) | (int(q) - 8));
}

struct KernelLaunch {
  const void* func;
  dim3 grid, block;
  size_t smem;
  int kind;
};

// TMA maps of the scratch buffers whose row count is that of the launch:
// one latent frame (M = B L rows), or all r_t sub-frames of the paper head's
// refinement blocks together (r_t M rows).
struct RowMaps {
  CUtensorMap q;            // Q [H][n_sub B][L][64]
  CUtensorMap o;            // attention output [rows][H Dh]
  CUtensorMap h;            // MLP hidden [rows][4D]
  CUtensorMap hs;           // spatial MLP hidden [rows][D] (paper head)
  CUtensorMap x8, h8;       // FP8 MLP operands [rows][D], [rows][4D]
};

// Where one Transformer block reads and writes: its residual stream (one
// latent frame, one sub-frame of the paper head, or all r_t sub-frames at
// once) and its ring cache.
struct BlockIO {
  float* x32;               // [M][D] fp32 residual stream (M rows)
  void* xb;                 // [M][D] storage-type copy (A operand)
  float* ssq;               // [M][D/32] sums of squares of x32
  const CUtensorMap* tm_x;  // map of xb (bf16 path)
  void* kc;                 // ring keys   [layers][B][G][kv_rows][Dh]
  void* vtc;                // ring values [layers][B][G][Dh][vt_pitch]
  int kv_rows, vt_pitch;
  const CUtensorMap* tm_k;  // maps over all layers of kc / vtc (bf16 path)
  const CUtensorMap* tm_v;
  int layer;                // this block's layer inside kc / vtc
  const FrameState* fs;     // state of stream 0, first (sub-)frame; stride fs_stride
  int M;                    // rows: n_sub sub-frames x B streams x L tokens
  int n_sub;                // sub-frames in one launch (1, or r_t)
  int kv_mirror;            // mirrored ring: rows between a key's two copies (0: none)
  int n_layers;             // layers of the ring (slabs of tm_k / tm_v: n_layers B G)
  int n_split;              // attention key splitting of this launch shape
  const RowMaps* maps;      // row-count-dependent maps (bf16 path)
};

// An attention node of the frame graph, kept so that its scratch pointers can
// be redirected (fd_decode_frame_static_scratch).
struct AttnNode {
  cudaGraphNode_t node = nullptr;
  KernelLaunch launch{};
  CUtensorMap tmQ{}, tmK{}, tmV{};
  TcAttnParams p{};
};

// A kernel node that writes the caller's pixel buffer (patched per call).
struct OutNode {
  cudaGraphNode_t node = nullptr;
  KernelLaunch launch{};
  EpiParams p{};
  CUtensorMap tmA{}, tmB{};
  const void* A = nullptr;
  const void* B = nullptr;
  int K = 0;
};

}  // namespace

// ============================================================== the handle
struct fd_handle {
  uint32_t magic = kMagic;
  fd_config cfg{};
  int bf = 0;                       // 1: bf16 storage + tcgen05 kernels
  int paper = 0;                    // 1: the paper's output head
  int fp8 = 0;                      // 1: FP8 E4M3 MLP GEMMs
  int tok_h = 0, tok_w = 0, L = 0, c_in = 0, qkv = 0, dff = 0, c_out = 0;
  int B = 1, M = 0;                 // video streams; GEMM rows M = B L
  int n_split = 1;                  // attention key splitting (1: off), one latent frame
  int n_split_ref = 1;              // the same for the batched refinement launches
  size_t split_units_max = 0;       // largest attention launch with splitting: units
  size_t split_rows_max = 0;        // and partial rows (units x n_split x 128)
  float *part_o = nullptr, *part_ml = nullptr;   // its partial results
  int* split_ctr = nullptr;
  int fs_stride = 1;                // FrameStates per stream: 1 (+ r_t, paper head)
  int kv_rows = 0, vt_pitch = 0, out_h = 0, out_w = 0, num_sms = 0;
  int device = -1;                  // the CUDA device the handle was created on
  int rkv_rows = 0, rvt_pitch = 0;  // refinement ring rows: ref_slots (x2 if mirrored) L
  // paper head: all r_t sub-frames pass each refinement block in one launch
  // per kernel (ref_batch), over a mirrored ring of ref_slots = r_t (W+2) - 1
  // sub-frames stored twice; otherwise sub-frame by sub-frame over a ring of
  // ref_slots = r_t (W+1)
  int ref_batch = 0, ref_slots = 0;
  int RM = 0;                       // rows of the largest launch: r_t M (ref_batch) or M
  size_t k_bytes = 0, v_bytes = 0, rk_bytes = 0, rv_bytes = 0;
  size_t latent_elems = 0, out_elems = 0, io_elt = 0, elt = 0;

  std::vector<void*> allocs;
  size_t dev_bytes = 0, cache_bytes = 0;

  float *embed_wT = nullptr, *embed_b = nullptr;
  std::vector<void*> wqkv, wo, w1, w2;
  std::vector<float*> bqkv, bo, b1, b2, gk, gv;
  void* wout = nullptr;
  float* bout = nullptr;
  void *wup = nullptr, *wsp1 = nullptr;     // paper head
  float *bup = nullptr, *bsp1 = nullptr;
  void *kc = nullptr, *vtc = nullptr;
  void *rkc = nullptr, *rvtc = nullptr;     // refinement ring (paper head)
  // FP8 MLP: per block (backbone, then refinement) static activation scales
  // and per-tensor weight scales; x8 = E4M3 image of the MLP-up's input
  // RMSNorm(x) / s_a; g2 = the RMSNorm gains before the MLP (fp32, also kept
  // for calibration, which records max |RMSNorm(x)|)
  std::vector<float> s_a, s_h, s_w1, s_w2;
  std::vector<float*> g2;
  void* x8 = nullptr;
  unsigned* amax = nullptr;                 // calibration: [blocks][2] float bits
  int n_amax = 0;
  float *x32 = nullptr, *ssq = nullptr;
  float *xs32 = nullptr, *xss = nullptr;    // [r_t][M][D], [r_t][M][D/32]
  void* xsb = nullptr;                      // [r_t][M][D] storage type
  void *xb = nullptr, *q = nullptr, *o = nullptr, *hb = nullptr;
  float2 *rope_row = nullptr, *rope_col = nullptr;
  double* inv_freq_t = nullptr;             // temporal RoPE frequencies theta^(-2m/d_t)
  long long* ctr = nullptr;
  FrameState* fs = nullptr;
  int* status = nullptr;
  // fd_decode_frame_host: two staging slots, so that the copy-out of frame t
  // (on the caller's stream) runs under the graph of frame t+1 (on host_stream)
  void* latent_stage[2] = {nullptr, nullptr};
  void* out_stage[2] = {nullptr, nullptr};
  cudaStream_t host_stream = nullptr;
  cudaEvent_t ev_graph[2] = {nullptr, nullptr};   // graph of the slot's frame done
  cudaEvent_t ev_d2h[2] = {nullptr, nullptr};     // copy-out of the slot's frame done
  cudaEvent_t ev_user = nullptr;                   // caller-stream work before a host call
  bool d2h_pending[2] = {false, false};
  int host_slot = 0;
  int g_last = -1;          // slot of the last graph on host_stream not yet joined
  bool user_pending = true; // caller-stream work since the last host call

  // TMA maps (bf16 path)
  CUtensorMap tm_xb{}, tm_k{}, tm_v{}, tm_wout{};
  CUtensorMap tm_rk{}, tm_rv{}, tm_wup{}, tm_wsp1{}, tm_xs_all{};
  RowMaps rm_frame{}, rm_ref{};        // M rows; r_t M rows (ref_batch)
  std::vector<CUtensorMap> tm_wqkv, tm_wo, tm_w1, tm_w2, tm_xs;

  // graph
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  cudaGraphNode_t last_node = nullptr;
  bool last_is_kernel = false;
  cudaGraphNode_t embed_node = nullptr;
  KernelLaunch embed_launch{};
  EmbedParams embed_p{};
  std::vector<OutNode> out_nodes;       // kernels writing the pixel buffer
  std::vector<AttnNode> attn_nodes;     // tcgen05 attention launches
  const void* cur_latent = nullptr;
  void* cur_out = nullptr;
  std::vector<cudaEvent_t> events;
  std::vector<int> kinds;               // fd_kernel_kind of every kernel node, in order
  struct Timed { int begin, end, kind; };
  std::vector<Timed> timed;             // kernels bracketed by event pairs
  cudaStream_t last_stream = nullptr;

  // ---------------------------------------------------------------- memory
  template <typename P>
  fd_status_t alloc(P** p, size_t bytes) {
    void* d = nullptr;
    cudaError_t e = cudaMalloc(&d, bytes ? bytes : 16);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(FD_ERR_OOM, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
    }
    allocs.push_back(d);
    dev_bytes += bytes;
    *p = static_cast<P*>(d);
    return FD_OK;
  }
  fd_status_t upload(void** dst, const void* src, size_t bytes) {
    FD_TRY(alloc(dst, bytes));
    FD_CUDA(cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice));
    return FD_OK;
  }
  fd_status_t upload_f32(float** dst, const float* src, size_t n) {
    void* d;
    FD_TRY(upload(&d, src, n * 4));
    *dst = static_cast<float*>(d);
    return FD_OK;
  }
  // Weight [rows][cols] with optional per-column gain folded in, quantized to
  // E4M3 with the per-tensor scale fp32(max|w g| / 448) (returned in *scale).
  fd_status_t upload_w_e4m3(void** dst, const float* w, size_t rows, size_t cols,
                            const float* gain, float* scale) {
    std::vector<double> v(rows * cols);
    double amax = 0.0;
    for (size_t r = 0; r < rows; ++r)
      for (size_t c = 0; c < cols; ++c) {
        v[r * cols + c] = double(w[r * cols + c]) * (gain ? double(gain[c]) : 1.0);
        amax = std::max(amax, std::fabs(v[r * cols + c]));
      }
    const float s = amax > 0.0 ? float(amax / 448.0) : 1.f;
    std::vector<uint8_t> q(rows * cols);
    for (size_t i = 0; i < q.size(); ++i) q[i] = e4m3_encode(v[i] / double(s));
    *scale = s;
    return upload(dst, q.data(), q.size());
  }
  // Weight [rows][cols] with optional per-column gain folded in, in storage type.
  fd_status_t upload_w(void** dst, const float* w, size_t rows, size_t cols, const float* gain) {
    if (bf) {
      std::vector<uint16_t> tmp(rows * cols);
      for (size_t r = 0; r < rows; ++r)
        for (size_t c = 0; c < cols; ++c) {
          const double v = double(w[r * cols + c]) * (gain ? double(gain[c]) : 1.0);
          tmp[r * cols + c] = f32_to_bf16_bits(float(v));
        }
      return upload(dst, tmp.data(), tmp.size() * 2);
    }
    std::vector<float> tmp(rows * cols);
    for (size_t r = 0; r < rows; ++r)
      for (size_t c = 0; c < cols; ++c)
        tmp[r * cols + c] = float(double(w[r * cols + c]) * (gain ? double(gain[c]) : 1.0));
    return upload(dst, tmp.data(), tmp.size() * 4);
  }

  ~fd_handle() {
    if (exec) cudaGraphExecDestroy(exec);
    if (graph) cudaGraphDestroy(graph);
    for (auto e : events) cudaEventDestroy(e);
    for (int i = 0; i < 2; ++i) {
      if (ev_graph[i]) cudaEventDestroy(ev_graph[i]);
      if (ev_d2h[i]) cudaEventDestroy(ev_d2h[i]);
    }
    if (ev_user) cudaEventDestroy(ev_user);
    if (host_stream) cudaStreamDestroy(host_stream);
    for (void* p : allocs) cudaFree(p);
  }

  // ---------------------------------------------------------------- graph
  fd_status_t add_event() {
    cudaEvent_t ev;
    FD_CUDA(cudaEventCreate(&ev));
    events.push_back(ev);
    cudaGraphNode_t n;
    FD_CUDA(cudaGraphAddEventRecordNode(&n, graph, last_node ? &last_node : nullptr,
                                        last_node ? 1 : 0, ev));
    last_node = n;
    last_is_kernel = false;
    return FD_OK;
  }
  // kernel_timing 1: one event after every kernel (consecutive events bracket
  // each kernel); 2: an event pair around each attention launch only.
  fd_status_t add_kernel(const KernelLaunch& k, void** args, cudaGraphNode_t* out_node = nullptr) {
    const bool bracket = cfg.kernel_timing == 2 && k.kind == FD_K_ATTN;
    int begin = int(events.size()) - 1;
    if (bracket) {
      FD_TRY(add_event());
      begin = int(events.size()) - 1;
    }
    cudaKernelNodeParams np{};
    np.func = const_cast<void*>(k.func);
    np.gridDim = k.grid;
    np.blockDim = k.block;
    np.sharedMemBytes = unsigned(k.smem);
    np.kernelParams = args;
    cudaGraphNode_t n;
    if (last_node && last_is_kernel && kUsePdl) {
      // programmatic edge: this kernel may launch once every CTA of the
      // previous one has started; its griddep_wait() orders the data
      FD_CUDA(cudaGraphAddKernelNode(&n, graph, nullptr, 0, &np));
      cudaGraphEdgeData edge{};
      edge.from_port = cudaGraphKernelNodePortProgrammatic;
      edge.type = cudaGraphDependencyTypeProgrammatic;
      FD_CUDA(cudaGraphAddDependencies_v2(graph, &last_node, &n, &edge, 1));
    } else {
      FD_CUDA(cudaGraphAddKernelNode(&n, graph, last_node ? &last_node : nullptr,
                                     last_node ? 1 : 0, &np));
    }
    last_node = n;
    last_is_kernel = true;
    if (out_node) *out_node = n;
    kinds.push_back(k.kind);
    if (cfg.kernel_timing == 1 || bracket) {
      FD_TRY(add_event());
      timed.push_back({begin, int(events.size()) - 1, k.kind});
    }
    return FD_OK;
  }

  fd_status_t build_graph();
  fd_status_t add_gemm(int kind, int fd_kind, const CUtensorMap& tmA, const void* A,
                       const CUtensorMap& tmB, const void* B, int N, int K, EpiParams ep,
                       cudaGraphNode_t* node, bool f8 = false);
  fd_status_t add_out_gemm(OutNode on, int N);
  fd_status_t add_block(int wi, const BlockIO& io);
  fd_status_t add_post_attention(int wi, const BlockIO& io);
  fd_status_t add_norm_quant(const BlockIO& io, int wi, float q_inv, unsigned* rec);
  EpiParams base_epi(const BlockIO& io) const;
  BlockIO backbone_io(int layer);
  BlockIO subframe_io(int tau, int layer);
  BlockIO refine_io(int layer);
};

namespace {

bool valid_handle(const fd_handle* h) { return h && h->magic == kMagic; }

// the longest CTA (64-key tiles over a full window) that the automatic
// choice gives one MMA-issuing thread (measured against 64: the XL paper
// head's refinement launches, 97 tiles, are 1.2% faster with one thread)
constexpr long kSingleIssuerMaxTiles = 100;


template <int BN, int KIND, bool F8>
fd_status_t tc_gemm_launch(int M, int N, int num_sms, KernelLaunch* k) {
  constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  using S = TcGemmSmem<BN, STAGES, KIND>;
  const void* f = reinterpret_cast<const void*>(&tc_gemm_kernel<BN, STAGES, KIND, 64, F8>);
  FD_CUDA(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc));
  const int tiles = ((M + 127) / 128) * (N / BN);
  k->func = f;
  k->grid = dim3(std::min(tiles, num_sms));
  k->block = dim3(gemm_threads(KIND));
  k->smem = S::kAlloc;
  return FD_OK;
}

// Tile width (BN) of a GEMM: the widest of 256 / 128 / 64 that divides N,
// except for the residual epilogues (O-projection, MLP-down). These are
// bound by their epilogue's memory latency. They switch to 128 when 256-wide
// tiles would occupy fewer CTAs than there are SMs and 128-wide tiles either
// still fit in one wave, or have a short K (<= 2048) and overflow the wave by
// at most 1/8. Measured faster for those shapes (480p: O-proj and MLP-down;
// FlashDecoder-XL 480p: O-proj), not faster for the others (720p O-proj at
// 1.57 waves, XL MLP-down with K = 6144, every 1080p GEMM). The weight tensor
// maps use the same rule for their box height.
int gemm_bn(int kind, int M, int N, int K, int num_sms) {
  if (N % 256 == 0) {
    const bool resid = kind == EPI_RESID || kind == EPI_RESID_Q;
    const long m_tiles = (M + 127) / 128;
    const long t256 = m_tiles * (N / 256), t128 = m_tiles * (N / 128);
    if (resid && t256 < num_sms &&
        (t128 <= num_sms || (K <= 2048 && t128 <= num_sms + num_sms / 8)))
      return 128;
    return 256;
  }
  return N % 128 == 0 ? 128 : 64;
}

template <int KIND, bool F8 = false>
fd_status_t tc_gemm_pick(int M, int N, int K, int num_sms, int* bn, KernelLaunch* k) {
  *bn = gemm_bn(KIND, M, N, K, num_sms);
  if (*bn == 256) return tc_gemm_launch<256, KIND, F8>(M, N, num_sms, k);
  if (*bn == 128) return tc_gemm_launch<128, KIND, F8>(M, N, num_sms, k);
  return tc_gemm_launch<64, KIND, F8>(M, N, num_sms, k);
}

template <int KIND>
const void* simt_gemm_fn(int dh) {
  return dh == 32 ? reinterpret_cast<const void*>(&simt_gemm_kernel<KIND, 32>)
                  : reinterpret_cast<const void*>(&simt_gemm_kernel<KIND, 64>);
}

}  // namespace

EpiParams fd_handle::base_epi(const BlockIO& io) const {
  EpiParams e{};
  e.M = io.M;
  e.L = L;
  e.B = B;
  e.fs_stride = fs_stride;
  e.out_stride = out_elems;
  e.ssq = io.ssq;
  e.ssq_parts = cfg.d_model / 32;
  e.inv_d = 1.f / float(cfg.d_model);
  e.eps = cfg.norm_eps;
  e.x32 = io.x32;
  e.xb = io.xb;
  e.ssq_out = io.ssq;
  e.D = cfg.d_model;
  e.q = q;
  e.H = cfg.n_heads;
  e.G = cfg.n_kv_heads;
  e.Dh = cfg.head_dim;
  e.kv_rows = io.kv_rows;
  e.vt_pitch = io.vt_pitch;
  e.kv_mirror = io.kv_mirror;
  e.kv_norm = cfg.kv_norm;
  e.fs = io.fs;
  e.rope_row = rope_row;
  e.rope_col = rope_col;
  e.tok_w = tok_w;
  e.tok_h = tok_h;
  e.P = cfg.px_per_token;
  e.out_bf16 = cfg.io_dtype == FD_BF16;
  e.pl_mul = 1;
  e.pl_add = 0;
  e.acc_scale = 1.f;
  e.q_inv = 1.f;
  e.status = status;
  e.n_sub = cfg.r_t;
  e.out_frames = cfg.out_ch * cfg.r_t;
  return e;
}

BlockIO fd_handle::backbone_io(int layer) {
  return BlockIO{x32, xb, ssq, &tm_xb, kc, vtc, kv_rows, vt_pitch, &tm_k, &tm_v, layer, fs,
                 M, 1, 0, cfg.n_blocks, n_split, &rm_frame};
}

// Sub-frame tau of the paper head through refinement layer `layer` alone.
BlockIO fd_handle::subframe_io(int tau, int layer) {
  const size_t rows = size_t(tau) * M;
  const int D = cfg.d_model;
  return BlockIO{xs32 + rows * D, static_cast<char*>(xsb) + rows * D * elt,
                 xss + rows * (D / 32), bf ? &tm_xs[tau] : &tm_xb, rkc, rvtc, rkv_rows,
                 rvt_pitch, &tm_rk, &tm_rv, layer, fs + 1 + tau,
                 M, 1, 0, cfg.n_refine, n_split, &rm_frame};
}

// All r_t sub-frames of the paper head through refinement layer `layer` in one
// launch per kernel (rows (tau B + b) L + n of xs), over the mirrored ring.
BlockIO fd_handle::refine_io(int layer) {
  return BlockIO{xs32, xsb, xss, &tm_xs_all, rkc, rvtc, rkv_rows, rvt_pitch, &tm_rk, &tm_rv,
                 layer, fs + 1, RM, cfg.r_t, ref_slots * L, cfg.n_refine, n_split_ref, &rm_ref};
}

// Kernel arguments must outlive the graph's construction; cudaGraphAddKernelNode
// copies the pointed-to values, so stack storage inside one call suffices.
fd_status_t fd_handle::add_gemm(int kind, int fd_kind, const CUtensorMap& tmA, const void* A,
                                const CUtensorMap& tmB, const void* B, int N, int K, EpiParams ep,
                                cudaGraphNode_t* node, bool f8) {
  ep.N = N;
  const int M = ep.M;
  KernelLaunch k{};
  if (bf) {
    int bn = 0;
    if (f8) {                     // FP8 MLP: the two MLP GEMMs
      if (kind == EPI_GELU_Q) FD_TRY((tc_gemm_pick<EPI_GELU_Q, true>(M, N, K, num_sms, &bn, &k)));
      else FD_TRY((tc_gemm_pick<EPI_RESID, true>(M, N, K, num_sms, &bn, &k)));
    } else switch (kind) {
      case EPI_QKV: FD_TRY(tc_gemm_pick<EPI_QKV>(M, N, K, num_sms, &bn, &k)); break;
      case EPI_RESID: FD_TRY(tc_gemm_pick<EPI_RESID>(M, N, K, num_sms, &bn, &k)); break;
      case EPI_GELU: FD_TRY(tc_gemm_pick<EPI_GELU>(M, N, K, num_sms, &bn, &k)); break;
      case EPI_UP: FD_TRY(tc_gemm_pick<EPI_UP>(M, N, K, num_sms, &bn, &k)); break;
      case EPI_RESID_Q: FD_TRY(tc_gemm_pick<EPI_RESID_Q>(M, N, K, num_sms, &bn, &k)); break;
      default: FD_TRY(tc_gemm_pick<EPI_FINAL>(M, N, K, num_sms, &bn, &k)); break;
    }
    CUtensorMap a = tmA, b = tmB;
    int kk = K;
    int* st = status;
    void* args[] = {&a, &b, &kk, &ep, &st};
    k.kind = fd_kind;
    return add_kernel(k, args, node);
  }
  switch (kind) {
    case EPI_QKV: k.func = simt_gemm_fn<EPI_QKV>(cfg.head_dim); break;
    case EPI_RESID: k.func = simt_gemm_fn<EPI_RESID>(cfg.head_dim); break;
    case EPI_GELU: k.func = simt_gemm_fn<EPI_GELU>(cfg.head_dim); break;
    case EPI_UP: k.func = simt_gemm_fn<EPI_UP>(cfg.head_dim); break;
    default: k.func = simt_gemm_fn<EPI_FINAL>(cfg.head_dim); break;
  }
  k.grid = dim3((M + 127) / 128, N / 64);
  k.block = dim3(128);
  k.smem = 0;
  k.kind = fd_kind;
  const float* a = static_cast<const float*>(A);
  const float* b = static_cast<const float*>(B);
  int kk = K;
  void* args[] = {&a, &b, &kk, &ep};
  return add_kernel(k, args, node);
}

// A FINAL GEMM whose output is the caller's pixel buffer; its launch and
// arguments are kept so that fd_decode_frame can point it at a new buffer.
fd_status_t fd_handle::add_out_gemm(OutNode on, int N) {
  on.p.N = N;
  FD_TRY(add_gemm(EPI_FINAL, FD_K_FINAL, on.tmA, on.A, on.tmB, on.B, N, on.K, on.p, &on.node));
  cudaKernelNodeParams np{};
  FD_CUDA(cudaGraphKernelNodeGetParams(on.node, &np));
  on.launch = KernelLaunch{np.func, np.gridDim, np.blockDim, np.sharedMemBytes, FD_K_FINAL};
  out_nodes.push_back(on);
  return FD_OK;
}

// One Transformer block (weights wi) on the stream and cache of io
// (paper Sec. 3.2-3.3): QKV (+RMSNorm, KV-norm, RoPE, ring write), window
// attention, O-projection (+residual), MLP-up (+RMSNorm, GELU), MLP-down
// (+residual).
fd_status_t fd_handle::add_block(int wi, const BlockIO& io) {
  const int D = cfg.d_model, H = cfg.n_heads, G = cfg.n_kv_heads, Dh = cfg.head_dim;
  void* kc_l = static_cast<char*>(io.kc) + size_t(io.layer) * B * G * io.kv_rows * Dh * elt;
  void* vtc_l = static_cast<char*>(io.vtc) + size_t(io.layer) * B * G * Dh * io.vt_pitch * elt;
  // QKV + KV-norm + RoPE + ring write
  EpiParams e = base_epi(io);
  e.bias = bqkv[wi];
  e.kc = kc_l;
  e.vtc = vtc_l;
  e.gk = gk[wi];
  e.gv = gv[wi];
  FD_TRY(add_gemm(EPI_QKV, FD_K_QKV, *io.tm_x, io.xb, bf ? tm_wqkv[wi] : *io.tm_x, wqkv[wi], qkv,
                  D, e, nullptr));
  // attention
  if (bf) {
    TcAttnParams ap{};
    ap.o = o;
    ap.L = L;
    ap.H = H;
    ap.G = G;
    ap.B = B;
    ap.n_sub = io.n_sub;
    ap.fs_stride = fs_stride;
    ap.layer = io.layer;
    ap.n_split = io.n_split;
    ap.part_o = part_o;
    ap.part_ml = part_ml;
    ap.counter = split_ctr;
    ap.scale_log2 = float(1.4426950408889634 / std::sqrt(double(Dh)));
    ap.fs = io.fs;
    ap.status = status;
    ap.kv_rows = io.kv_rows;
    ap.n_slabs = io.n_layers * B * G;
    // one MMA-issuing thread for launches that fill every CTA slot (2 per SM)
    // at least once with CTAs of at most 100 key tiles (full window); two
    // otherwise. Measured: 1.5-3.4% faster attention at 720p (56 tiles per
    // CTA) and for the XL shapes (16-98); 2% slower at 480p (208 CTAs for 296
    // slots); at 1080p (128-192 tiles) 0.6% fewer cycles per frame but a
    // 1.2% lower clock under the 1000 W power cap, a net loss
    const long ctas = long((L + 127) / 128) * H * io.n_sub * B * io.n_split;
    const long window_keys = long(io.kv_mirror ? cfg.r_t * (cfg.window + 1) : io.kv_rows / L) * L;
    const long tiles = (window_keys + 63) / 64 / io.n_split;
    ap.single_issuer = cfg.attn_issuer == 2 ||
                       (cfg.attn_issuer == 0 && ctas >= 2L * num_sms && tiles <= kSingleIssuerMaxTiles);
    // one 128-query tile per CTA, two CTAs per SM (measured faster than two
    // query tiles sharing one CTA, and than three CTAs with single-buffered S)
    using A = TcAttnSmem;
    const void* f = reinterpret_cast<const void*>(&tc_attn_kernel);
    FD_CUDA(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, A::kAlloc));
    KernelLaunch k{f, dim3((L + 127) / 128, H, io.n_sub * B * io.n_split), dim3(A::kThreads),
                   size_t(A::kAlloc), FD_K_ATTN};
    CUtensorMap a = io.maps->q, b = *io.tm_k, c = *io.tm_v;
    void* args[] = {&a, &b, &c, &ap};
    AttnNode an;
    FD_TRY(add_kernel(k, args, &an.node));
    an.launch = k;
    an.tmQ = a;
    an.tmK = b;
    an.tmV = c;
    an.p = ap;
    attn_nodes.push_back(an);
  } else {
    AttnParams ap{};
    ap.q = q;
    ap.kc = kc_l;
    ap.vtc = vtc_l;
    ap.o = o;
    ap.L = L;
    ap.H = H;
    ap.G = G;
    ap.kv_rows = io.kv_rows;
    ap.vt_pitch = io.vt_pitch;
    ap.B = B;
    ap.fs_stride = fs_stride;
    ap.scale_log2 = float(1.4426950408889634 / std::sqrt(double(Dh)));
    ap.fs = io.fs;
    ap.status = status;
    const void* f = Dh == 32 ? reinterpret_cast<const void*>(&simt_attn_kernel<32>)
                             : reinterpret_cast<const void*>(&simt_attn_kernel<64>);
    KernelLaunch k{f, dim3((L + 63) / 64, H, B), dim3(64), 0, FD_K_ATTN};
    void* args[] = {&ap};
    FD_TRY(add_kernel(k, args));
  }
  return add_post_attention(wi, io);
}

// The rest of a block after its attention: O-projection (+residual), MLP-up
// (+RMSNorm, GELU), MLP-down (+residual); FP8 E4M3 MLP with mlp_fp8.
fd_status_t fd_handle::add_post_attention(int wi, const BlockIO& io) {
  const int D = cfg.d_model, H = cfg.n_heads, Dh = cfg.head_dim;
  EpiParams e;
  if (fp8) {
    // output projection + residual (x32 and its sums of squares only)
    e = base_epi(io);
    e.bias = bo[wi];
    FD_TRY(add_gemm(EPI_RESID_Q, FD_K_OPROJ, io.maps->o, o, tm_wo[wi], wo[wi], D, H * Dh, e,
                    nullptr));
    // the MLP-up's input: x8 = e4m3(RMSNorm(x) / s_a)
    FD_TRY(add_norm_quant(io, wi, float(1.0 / double(s_a[wi])), nullptr));
    // FP8 MLP up: h = GELU((x8 W1q^T) s_a s_w1 + b_1) stored as e4m3(h / s_h)
    e = base_epi(io);
    e.bias = b1[wi];
    e.hout = hb;
    e.acc_scale = float(double(s_a[wi]) * double(s_w1[wi]));
    e.q_inv = float(1.0 / double(s_h[wi]));
    FD_TRY(add_gemm(EPI_GELU_Q, FD_K_MLP_UP, io.maps->x8, x8, tm_w1[wi], w1[wi], dff, D, e,
                    nullptr, true));
    // FP8 MLP down + residual: x += (h8 W2q^T) s_h s_w2 + b_2
    e = base_epi(io);
    e.bias = b2[wi];
    e.acc_scale = float(double(s_h[wi]) * double(s_w2[wi]));
    return add_gemm(EPI_RESID, FD_K_MLP_DOWN, io.maps->h8, hb, tm_w2[wi], w2[wi], D, dff, e,
                    nullptr, true);
  }
  // output projection + residual
  e = base_epi(io);
  e.bias = bo[wi];
  FD_TRY(add_gemm(EPI_RESID, FD_K_OPROJ, io.maps->o, o, bf ? tm_wo[wi] : io.maps->o, wo[wi], D,
                  H * Dh, e, nullptr));
  // calibration: max |RMSNorm(x)| entering the MLP
  if (amax) FD_TRY(add_norm_quant(io, wi, 1.f, amax + 2 * wi));
  // MLP up + GELU
  e = base_epi(io);
  e.bias = b1[wi];
  e.hout = hb;
  if (amax) e.amax = amax + 2 * wi + 1;           // calibration: max |GELU output|
  FD_TRY(add_gemm(EPI_GELU, FD_K_MLP_UP, *io.tm_x, io.xb, bf ? tm_w1[wi] : *io.tm_x, w1[wi], dff,
                  D, e, nullptr));
  // MLP down + residual
  e = base_epi(io);
  e.bias = b2[wi];
  return add_gemm(EPI_RESID, FD_K_MLP_DOWN, io.maps->h, hb, bf ? tm_w2[wi] : io.maps->h, w2[wi],
                  D, dff, e, nullptr);
}

// RMSNorm(x) of the MLP's input (gain of block wi): its E4M3 image
// e4m3(a q_inv) into x8 (FP8 MLP), or with rec set its max |a| (calibration).
fd_status_t fd_handle::add_norm_quant(const BlockIO& io, int wi, float q_inv, unsigned* rec) {
  NormQuantParams np{};
  np.x32 = io.x32;
  np.ssq = io.ssq;
  np.g = g2[wi];
  np.x8 = rec ? nullptr : static_cast<uint8_t*>(x8);
  np.amax = rec;
  np.M = io.M;
  np.D = cfg.d_model;
  np.inv_d = 1.f / float(cfg.d_model);
  np.eps = cfg.norm_eps;
  np.q_inv = q_inv;
  KernelLaunch k{reinterpret_cast<const void*>(&mlp_norm_quant_kernel), dim3((io.M + 7) / 8),
                 dim3(256), 0, FD_K_MLP_NORM};
  void* args[] = {&np};
  return add_kernel(k, args);
}

fd_status_t fd_handle::build_graph() {
  FD_CUDA(cudaGraphCreate(&graph, 0));
  last_node = nullptr;
  last_is_kernel = false;
  if (cfg.kernel_timing == 1) FD_TRY(add_event());

  // step_begin
  {
    KernelLaunch k{reinterpret_cast<const void*>(&step_begin_kernel), dim3(1), dim3(256), 0,
                   FD_K_STEP_BEGIN};
    long long* c = ctr;
    FrameState* f = fs;
    int W = cfg.window, pairs = cfg.head_dim / 8, n_sub = paper ? cfg.r_t : 0, nb = B;
    int sub_cap = paper ? ref_slots : 1, sub_mirror = ref_batch;
    const double* fr = inv_freq_t;
    void* args[] = {&c, &f, &W, &pairs, &fr, &n_sub, &nb, &sub_cap, &sub_mirror};
    FD_TRY(add_kernel(k, args));
  }
  // embed
  {
    embed_p.latent = latent_stage[0];
    embed_p.latent_bf16 = cfg.io_dtype == FD_BF16;
    embed_p.C = cfg.latent_ch;
    embed_p.Hl = cfg.grid_h;
    embed_p.Wl = cfg.grid_w;
    embed_p.p = cfg.patch;
    embed_p.tok_w = tok_w;
    embed_p.L = L;
    embed_p.M = M;
    embed_p.c_in = c_in;
    embed_p.wT = embed_wT;
    embed_p.b = embed_b;
    embed_p.D = cfg.d_model;
    embed_p.x32 = x32;
    embed_p.xb = xb;
    embed_p.ssq = ssq;
    embed_p.status = status;
    const void* f = bf ? reinterpret_cast<const void*>(&embed_kernel<bf16>)
                       : reinterpret_cast<const void*>(&embed_kernel<float>);
    embed_launch = KernelLaunch{f, dim3((M + kEmbedTok - 1) / kEmbedTok), dim3(kEmbedThreads),
                                size_t(kEmbedTok) * c_in * 4, FD_K_EMBED};
    void* args[] = {&embed_p};
    FD_TRY(add_kernel(embed_launch, args, &embed_node));
    cur_latent = latent_stage[0];
  }
  const int D = cfg.d_model;
  for (int l = 0; l < cfg.n_blocks; ++l) FD_TRY(add_block(l, backbone_io(l)));

  if (!paper) {
    // final norm + projection + unpatchify
    OutNode on;
    on.p = base_epi(backbone_io(0));
    on.p.bias = bout;
    on.p.out = out_stage[0];
    on.tmA = tm_xb;
    on.A = xb;
    on.tmB = bf ? tm_wout : tm_xb;
    on.B = wout;
    on.K = D;
    FD_TRY(add_out_gemm(on, c_out));
  } else {
    // temporal upsampling (Eq. 3): xs[tau] = (up_w x + up_b)[tau D, (tau+1) D)
    EpiParams e = base_epi(backbone_io(0));
    e.bias = bup;
    e.ssq = nullptr;
    e.x32 = xs32;
    e.xb = xsb;
    e.ssq_out = xss;
    FD_TRY(add_gemm(EPI_UP, FD_K_UPSAMPLE, tm_xb, xb, bf ? tm_wup : tm_xb, wup, cfg.r_t * D, D, e,
                    nullptr));
    const int c_px = cfg.out_ch * cfg.px_per_token * cfg.px_per_token;
    // spatial MLP (layer 1: GELU(RMSNorm(xs) sp1_w^T + sp1_b) -> hidden; layer
    // 2 + PixelShuffle into pixel frames (c, tau), no norm) of the rows of io
    auto spatial = [&](const BlockIO& io, int tau) -> fd_status_t {
      EpiParams es = base_epi(io);
      es.bias = bsp1;
      es.hout = hb;
      FD_TRY(add_gemm(EPI_GELU, FD_K_SPATIAL, *io.tm_x, io.xb, bf ? tm_wsp1 : *io.tm_x, wsp1, D,
                      D, es, nullptr));
      OutNode on;
      on.p = base_epi(io);
      on.p.bias = bout;
      on.p.ssq = nullptr;
      on.p.out = out_stage[0];
      on.p.pl_mul = cfg.r_t;
      on.p.pl_add = tau;                  // 0 for a batched launch: tau comes from the row
      on.tmA = bf ? io.maps->hs : tm_xb;
      on.A = hb;
      on.tmB = bf ? tm_wout : tm_xb;
      on.B = wout;
      on.K = D;
      return add_out_gemm(on, c_px);
    };
    if (ref_batch) {
      // every refinement block once over all r_t sub-frames (r_t M rows), then
      // the spatial MLP over all of them
      for (int l = 0; l < cfg.n_refine; ++l) FD_TRY(add_block(cfg.n_blocks + l, refine_io(l)));
      FD_TRY(spatial(refine_io(0), 0));
    } else {
      for (int tau = 0; tau < cfg.r_t; ++tau) {
        // refinement blocks: sub-frame t r_t + tau in the ring of r_t (W+1)
        for (int l = 0; l < cfg.n_refine; ++l)
          FD_TRY(add_block(cfg.n_blocks + l, subframe_io(tau, l)));
        FD_TRY(spatial(subframe_io(tau, 0), tau));
      }
    }
  }
  cur_out = out_stage[0];
  FD_CUDA(cudaGraphInstantiate(&exec, graph, 0));
  return FD_OK;
}

// ============================================================== C ABI
namespace {

fd_status_t validate(const fd_config* c) {
  if (c->latent_ch <= 0 || c->grid_h <= 0 || c->grid_w <= 0 || c->d_model <= 0 ||
      c->n_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 || c->n_blocks <= 0 ||
      c->mlp_ratio <= 0 || c->window < 0 || c->out_ch <= 0 || c->r_t <= 0 ||
      c->px_per_token <= 0)
    return fail(FD_ERR_INVALID_ARG, "config: every size must be positive (window >= 0)");
  if (c->patch != 1 && c->patch != 2)
    return fail(FD_ERR_UNSUPPORTED, "config: patch must be 1 or 2 (got %d)", c->patch);
  if (c->grid_h % c->patch || c->grid_w % c->patch)
    return fail(FD_ERR_INVALID_ARG, "config: latent grid %dx%d not divisible by patch %d",
                c->grid_h, c->grid_w, c->patch);
  if (c->n_heads % c->n_kv_heads)
    return fail(FD_ERR_INVALID_ARG, "config: n_kv_heads (%d) must divide n_heads (%d)",
                c->n_kv_heads, c->n_heads);
  if (c->dtype != FD_F32 && c->dtype != FD_BF16)
    return fail(FD_ERR_INVALID_ARG, "config: unknown dtype %d", int(c->dtype));
  if (c->io_dtype != FD_F32 && c->io_dtype != FD_BF16)
    return fail(FD_ERR_INVALID_ARG, "config: unknown io_dtype %d", int(c->io_dtype));
  if (c->kv_norm != 0 && c->kv_norm != 1)
    return fail(FD_ERR_INVALID_ARG, "config: kv_norm must be 0 or 1");
  if (!(c->norm_eps > 0.f) || !(c->rope_theta > 1.f))
    return fail(FD_ERR_INVALID_ARG, "config: norm_eps must be > 0 and rope_theta > 1");
  if (c->px_per_token != 8 && c->px_per_token != 16)
    return fail(FD_ERR_UNSUPPORTED, "config: px_per_token must be 8 or 16");
  if (c->d_model % 64)
    return fail(FD_ERR_UNSUPPORTED, "config: d_model must be a multiple of 64");
  const int qkv = (c->n_heads + 2 * c->n_kv_heads) * c->head_dim;
  if (c->dtype == FD_BF16) {
    if (c->head_dim != 64)
      return fail(FD_ERR_UNSUPPORTED, "config: bf16 kernels need head_dim 64 (got %d)",
                  c->head_dim);
  } else {
    if (c->head_dim != 32 && c->head_dim != 64)
      return fail(FD_ERR_UNSUPPORTED, "config: head_dim must be 32 or 64 (got %d)", c->head_dim);
    if (qkv % 64 || (c->n_heads * c->head_dim) % 32)
      return fail(FD_ERR_UNSUPPORTED, "config: (N+2G)*D_h must be a multiple of 64");
  }
  const long long L = (long long)(c->grid_h / c->patch) * (c->grid_w / c->patch);
  if (L * (c->window + 1) > (1LL << 30))
    return fail(FD_ERR_UNSUPPORTED, "config: window of %lld tokens is too large",
                L * (c->window + 1));
  if (c->attn_splits < 0 || c->attn_splits > 4)
    return fail(FD_ERR_INVALID_ARG, "config: attn_splits must be 0 .. 4 (got %d)", c->attn_splits);
  if (c->attn_issuer < 0 || c->attn_issuer > 2)
    return fail(FD_ERR_INVALID_ARG, "config: attn_issuer must be 0 .. 2 (got %d)", c->attn_issuer);
  if (c->batch < 1 || c->batch > fd::kMaxStreams)
    return fail(FD_ERR_INVALID_ARG, "config: batch must be 1 .. %d (got %d)", fd::kMaxStreams, c->batch);
  if (c->kernel_timing < 0 || c->kernel_timing > 2)
    return fail(FD_ERR_INVALID_ARG, "config: kernel_timing must be 0, 1 or 2");
  if (c->head_mode != 0 && c->head_mode != 1)
    return fail(FD_ERR_INVALID_ARG, "config: head_mode must be 0 or 1");
  if ((c->mlp_fp8 != 0 && c->mlp_fp8 != 1) || (c->record_mlp_amax != 0 && c->record_mlp_amax != 1))
    return fail(FD_ERR_INVALID_ARG, "config: mlp_fp8 and record_mlp_amax must be 0 or 1");
  if (c->record_mlp_amax && c->d_model % 128)
    return fail(FD_ERR_UNSUPPORTED, "config: record_mlp_amax needs d_model a multiple of 128");
  if (c->mlp_fp8 && (c->dtype != FD_BF16 || c->d_model % 128))
    return fail(FD_ERR_UNSUPPORTED, "config: mlp_fp8 needs dtype bf16 and d_model a multiple of 128");
  if (c->mlp_fp8 && c->record_mlp_amax)
    return fail(FD_ERR_INVALID_ARG, "config: record_mlp_amax calibrates the unquantized MLP (mlp_fp8 0)");
  if (c->head_mode == 1) {
    if (c->n_refine < 1 || c->n_refine > 8)
      return fail(FD_ERR_UNSUPPORTED, "config: n_refine must be 1 .. 8 (got %d)", c->n_refine);
    if (c->r_t > 16)
      return fail(FD_ERR_UNSUPPORTED, "config: the paper head supports r_t <= 16 (got %d)", c->r_t);
    // ring rows: r_t (W+1) sub-frames, or 2 (r_t (W+2) - 1) when mirrored
    const long long ring = (c->dtype == FD_BF16 && L % 8 == 0)
                               ? 2LL * (c->r_t * (c->window + 2) - 1) * L
                               : L * c->r_t * (c->window + 1);
    if (ring > (1LL << 30))
      return fail(FD_ERR_UNSUPPORTED, "config: refinement ring of %lld tokens is too large", ring);
  }
  return FD_OK;
}

fd_status_t create_impl(const fd_config* cfg, const fd_weights* w, fd_handle* h) {
  h->cfg = *cfg;
  const fd_config& c = *cfg;
  h->bf = c.dtype == FD_BF16;
  h->paper = c.head_mode == 1;
  h->fp8 = c.mlp_fp8;
  h->elt = h->bf ? 2 : 4;
  h->io_elt = c.io_dtype == FD_BF16 ? 2 : 4;
  h->tok_h = c.grid_h / c.patch;
  h->tok_w = c.grid_w / c.patch;
  h->L = h->tok_h * h->tok_w;
  h->B = c.batch;
  h->M = h->B * h->L;
  h->fs_stride = 1 + (c.head_mode == 1 ? c.r_t : 0);
  h->c_in = c.latent_ch * c.patch * c.patch;
  h->qkv = (c.n_heads + 2 * c.n_kv_heads) * c.head_dim;
  h->dff = c.mlp_ratio * c.d_model;
  h->c_out = c.out_ch * c.r_t * c.px_per_token * c.px_per_token;
  h->kv_rows = (c.window + 1) * h->L;
  h->vt_pitch = int(round_up(size_t(h->kv_rows), 64));
  // paper head, bf16: the r_t sub-frames go through each refinement block in
  // one launch per kernel, over a mirrored ring (every window a contiguous key
  // range). The TMA load of the transposed values starts at key win * L, which
  // must be a multiple of 8 (16 bytes), hence L % 8 == 0; otherwise, and on
  // the fp32 path, sub-frame by sub-frame.
  h->ref_batch = h->paper && h->bf && h->L % 8 == 0;
  h->ref_slots = h->ref_batch ? c.r_t * (c.window + 2) - 1 : c.r_t * (c.window + 1);
  h->rkv_rows = (h->ref_batch ? 2 : 1) * h->ref_slots * h->L;
  h->rvt_pitch = int(round_up(size_t(h->rkv_rows), 64));
  h->RM = h->ref_batch ? c.r_t * h->M : h->M;
  h->out_h = h->tok_h * c.px_per_token;
  h->out_w = h->tok_w * c.px_per_token;
  h->latent_elems = size_t(c.latent_ch) * c.grid_h * c.grid_w;
  h->out_elems = size_t(c.out_ch) * c.r_t * h->out_h * h->out_w;
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev));
  h->device = dev;
  int major = 0;
  FD_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  FD_CUDA(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));
  if (major != 10)
    return fail(FD_ERR_UNSUPPORTED, "device compute capability %d.x: this library is built for sm_100a",
                major);

  const int D = c.d_model, H = c.n_heads, G = c.n_kv_heads, Dh = c.head_dim, NB = c.n_blocks;
  const int NR = h->paper ? c.n_refine : 0;        // refinement blocks follow the backbone's
  const int c_px = c.out_ch * c.px_per_token * c.px_per_token;
  // ---- weights
  {
    std::vector<float> wT(size_t(h->c_in) * D);
    for (int d = 0; d < D; ++d)
      for (int ch = 0; ch < h->c_in; ++ch) wT[size_t(ch) * D + d] = w->embed_w[size_t(d) * h->c_in + ch];
    FD_TRY(h->upload_f32(&h->embed_wT, wT.data(), wT.size()));
    FD_TRY(h->upload_f32(&h->embed_b, w->embed_b, D));
  }
  std::vector<float> ones(std::max(D, Dh), 1.f);
  for (int l = 0; l < NB + NR; ++l) {
    void* p;
    FD_TRY(h->upload_w(&p, w->wqkv[l], h->qkv, D, w->norm1_g[l])); h->wqkv.push_back(p);
    FD_TRY(h->upload_w(&p, w->wo[l], D, size_t(H) * Dh, nullptr)); h->wo.push_back(p);
    if (h->fp8) {
      float s1 = 1.f, s2 = 1.f;
      FD_TRY(h->upload_w_e4m3(&p, w->w1[l], h->dff, D, nullptr, &s1)); h->w1.push_back(p);
      FD_TRY(h->upload_w_e4m3(&p, w->w2[l], D, h->dff, nullptr, &s2)); h->w2.push_back(p);
      h->s_w1.push_back(s1);
      h->s_w2.push_back(s2);
      h->s_a.push_back(w->mlp_scales[l][0]);
      h->s_h.push_back(w->mlp_scales[l][1]);
    } else {
      FD_TRY(h->upload_w(&p, w->w1[l], h->dff, D, w->norm2_g[l])); h->w1.push_back(p);
      FD_TRY(h->upload_w(&p, w->w2[l], D, h->dff, nullptr)); h->w2.push_back(p);
    }
    float* f;
    if (h->fp8 || c.record_mlp_amax) {
      FD_TRY(h->upload_f32(&f, w->norm2_g[l], D)); h->g2.push_back(f);
    }
    FD_TRY(h->upload_f32(&f, w->bqkv[l], h->qkv)); h->bqkv.push_back(f);
    FD_TRY(h->upload_f32(&f, w->bo[l], D)); h->bo.push_back(f);
    FD_TRY(h->upload_f32(&f, w->b1[l], h->dff)); h->b1.push_back(f);
    FD_TRY(h->upload_f32(&f, w->b2[l], D)); h->b2.push_back(f);
    FD_TRY(h->upload_f32(&f, c.kv_norm ? w->knorm_g[l] : ones.data(), Dh)); h->gk.push_back(f);
    FD_TRY(h->upload_f32(&f, c.kv_norm ? w->vnorm_g[l] : ones.data(), Dh)); h->gv.push_back(f);
  }
  if (!h->paper) {
    FD_TRY(h->upload_w(&h->wout, w->out_w, h->c_out, D, w->final_g));
    FD_TRY(h->upload_f32(&h->bout, w->out_b, h->c_out));
  } else {
    // final_g is the RMSNorm before the spatial MLP: folded into its first layer
    FD_TRY(h->upload_w(&h->wup, w->up_w, size_t(c.r_t) * D, D, nullptr));
    FD_TRY(h->upload_f32(&h->bup, w->up_b, size_t(c.r_t) * D));
    FD_TRY(h->upload_w(&h->wsp1, w->sp1_w, D, D, w->final_g));
    FD_TRY(h->upload_f32(&h->bsp1, w->sp1_b, D));
    FD_TRY(h->upload_w(&h->wout, w->out_w, c_px, D, nullptr));
    FD_TRY(h->upload_f32(&h->bout, w->out_b, c_px));
  }

  // ---- ring caches: K [layers][B][G][rows][Dh], V^T [layers][B][G][Dh][pitch];
  // backbone rows = (W+1) L, refinement rows = ref_slots L (x2 when mirrored)
  const int BG = h->B * G;
  h->k_bytes = size_t(NB) * BG * h->kv_rows * Dh * h->elt;
  h->v_bytes = size_t(NB) * BG * Dh * h->vt_pitch * h->elt;
  FD_TRY(h->alloc(&h->kc, h->k_bytes));
  FD_TRY(h->alloc(&h->vtc, h->v_bytes));
  if (h->paper) {
    h->rk_bytes = size_t(NR) * BG * h->rkv_rows * Dh * h->elt;
    h->rv_bytes = size_t(NR) * BG * Dh * h->rvt_pitch * h->elt;
    FD_TRY(h->alloc(&h->rkc, h->rk_bytes));
    FD_TRY(h->alloc(&h->rvtc, h->rv_bytes));
  }
  h->cache_bytes = h->k_bytes + h->v_bytes + h->rk_bytes + h->rv_bytes;

  // ---- scratch
  const size_t L = h->M;                 // every per-frame buffer holds B frames
  const size_t RM = h->RM;               // the buffers a batched refinement launch
  FD_TRY(h->alloc(&h->x32, L * D * 4));  // uses hold its r_t M rows
  FD_TRY(h->alloc(&h->xb, L * D * h->elt));
  FD_TRY(h->alloc(&h->ssq, L * (D / 32) * 4));
  FD_TRY(h->alloc(&h->q, size_t(H) * RM * Dh * h->elt));
  FD_TRY(h->alloc(&h->o, RM * H * Dh * h->elt));
  FD_TRY(h->alloc(&h->hb, RM * h->dff * h->elt));
  if (h->paper) {
    FD_TRY(h->alloc(&h->xs32, size_t(c.r_t) * L * D * 4));
    FD_TRY(h->alloc(&h->xsb, size_t(c.r_t) * L * D * h->elt));
    FD_TRY(h->alloc(&h->xss, size_t(c.r_t) * L * (D / 32) * 4));
  }
  if (h->fp8) FD_TRY(h->alloc(&h->x8, RM * D));
  if (c.record_mlp_amax) {
    h->n_amax = 2 * (NB + NR);
    FD_TRY(h->alloc(&h->amax, size_t(h->n_amax) * 4));
  }
  // attention key splitting, per launch shape (one latent frame; all r_t
  // sub-frames of a batched refinement block): chosen by the launch's fit to
  // the CTA slots (2 per SM): est(s) = waves(s units) / s, plus 4% per extra
  // split for the partial writes and the combine. One scratch serves both
  // shapes (their launches never overlap), sized for the larger.
  if (h->bf) {
    const long slots = 2L * h->num_sms;
    auto pick = [&](long units) {
      int ns = c.attn_splits;
      if (ns == 0) {
        double best = 1e30;
        for (int sp = 1; sp <= 3; ++sp) {
          const double est = double((units * sp + slots - 1) / slots) / sp * (1.0 + 0.04 * (sp - 1));
          if (est < best - 1e-9) { best = est; ns = sp; }
        }
      }
      if (ns > 1) {
        h->split_units_max = std::max(h->split_units_max, size_t(units));
        h->split_rows_max = std::max(h->split_rows_max, size_t(units) * ns * 128);
      }
      return ns;
    };
    const long units = long((h->L + 127) / 128) * H * h->B;
    h->n_split = pick(units);
    h->n_split_ref = h->ref_batch ? pick(units * c.r_t) : h->n_split;
    if (h->split_rows_max > 0) {
      FD_TRY(h->alloc(&h->part_o, h->split_rows_max * 64 * 4));
      FD_TRY(h->alloc(&h->part_ml, h->split_rows_max * 2 * 4));
      FD_TRY(h->alloc(&h->split_ctr, h->split_units_max * 4));
      FD_CUDA(cudaMemset(h->split_ctr, 0, h->split_units_max * 4));
    }
  }
  FD_TRY(h->alloc(&h->ctr, size_t(h->B) * 8));
  FD_TRY(h->alloc(&h->fs, sizeof(FrameState) * h->fs_stride * h->B));
  FD_TRY(h->alloc(&h->status, 16));
  for (int i = 0; i < 2; ++i) {
    FD_TRY(h->alloc(&h->latent_stage[i], round_up(h->B * h->latent_elems * h->io_elt, 256)));
    FD_TRY(h->alloc(&h->out_stage[i], round_up(h->B * h->out_elems * h->io_elt, 256)));
    FD_CUDA(cudaEventCreateWithFlags(&h->ev_graph[i], cudaEventDisableTiming));
    FD_CUDA(cudaEventCreateWithFlags(&h->ev_d2h[i], cudaEventDisableTiming));
  }
  FD_CUDA(cudaEventCreateWithFlags(&h->ev_user, cudaEventDisableTiming));
  FD_CUDA(cudaStreamCreateWithFlags(&h->host_stream, cudaStreamNonBlocking));

  // ---- temporal RoPE frequencies (fp64): d_t = D_h / 4 dims, pair m at
  // theta^(-2m/d_t); the angles themselves depend on the frame counter and are
  // formed on the device by step_begin
  {
    const int dt = Dh / 4;
    std::vector<double> fr(dt / 2);
    for (int m = 0; m < dt / 2; ++m) fr[m] = std::pow(double(c.rope_theta), -2.0 * m / dt);
    void* p;
    FD_TRY(h->upload(&p, fr.data(), fr.size() * sizeof(double)));
    h->inv_freq_t = static_cast<double*>(p);
  }
  // ---- spatial RoPE tables (fp64 angles): row part and column part,
  // d_s = 3 D_h / 8 dims each, pair m at frequency theta^(-2m/d_s)
  {
    const int ds = 3 * Dh / 8;
    std::vector<float2> rr(size_t(h->tok_h) * (ds / 2)), rc(size_t(h->tok_w) * (ds / 2));
    for (int i = 0; i < h->tok_h; ++i)
      for (int m = 0; m < ds / 2; ++m) {
        const double a = i * std::pow(double(c.rope_theta), -2.0 * m / ds);
        rr[size_t(i) * (ds / 2) + m] = make_float2(float(std::cos(a)), float(std::sin(a)));
      }
    for (int j = 0; j < h->tok_w; ++j)
      for (int m = 0; m < ds / 2; ++m) {
        const double a = j * std::pow(double(c.rope_theta), -2.0 * m / ds);
        rc[size_t(j) * (ds / 2) + m] = make_float2(float(std::cos(a)), float(std::sin(a)));
      }
    void* p;
    FD_TRY(h->upload(&p, rr.data(), rr.size() * sizeof(float2))); h->rope_row = static_cast<float2*>(p);
    FD_TRY(h->upload(&p, rc.data(), rc.size() * sizeof(float2))); h->rope_col = static_cast<float2*>(p);
  }

  // ---- tensor maps (bf16 path)
  if (h->bf) {
    FD_TRY(make_tmap_2d(&h->tm_xb, h->xb, L, D, 128));
    // maps of the buffers whose rows are those of the launch: one latent frame
    // (M rows), and for batched refinement all r_t sub-frames (r_t M rows)
    auto row_maps = [&](RowMaps* rm, size_t rows, int n_sub) -> fd_status_t {
      FD_TRY(make_tmap_2d(&rm->o, h->o, rows, size_t(H) * Dh, 128));
      FD_TRY(make_tmap_2d(&rm->h, h->hb, rows, h->dff, 128));
      if (h->paper) FD_TRY(make_tmap_2d(&rm->hs, h->hb, rows, D, 128));   // spatial hidden
      if (h->fp8) {
        FD_TRY(make_tmap_2d_e4m3(&rm->x8, h->x8, rows, D, 128));
        FD_TRY(make_tmap_2d_e4m3(&rm->h8, h->hb, rows, h->dff, 128));   // hidden as E4M3
      }
      // Q [H][n_sub B][L_frm][64]: box 64 x 128 x 1 x 1; a stream's last tile reads zeros
      const uint64_t Lf = uint64_t(h->L), nb = uint64_t(n_sub) * h->B;
      const uint64_t dims[4] = {64, Lf, nb, uint64_t(H)};
      const uint64_t str[3] = {64 * 2, Lf * 64 * 2, nb * Lf * 64 * 2};
      const uint32_t box[4] = {64, 128, 1, 1};
      return make_tmap(&rm->q, h->q, 4, dims, str, box);
    };
    FD_TRY(row_maps(&h->rm_frame, L, 1));
    if (h->ref_batch) FD_TRY(row_maps(&h->rm_ref, RM, c.r_t));
    // a weight map's box is the BN rows its GEMM's tile width takes, which
    // depends on the launch's row count
    auto bn_of = [&](size_t rows, int N, int kind = EPI_QKV, int K = 0) {
      return uint32_t(gemm_bn(kind, int(rows), N, K, h->num_sms));
    };
    for (int l = 0; l < NB + NR; ++l) {
      const size_t rows = l < NB ? L : RM;
      CUtensorMap m;
      FD_TRY(make_tmap_2d(&m, h->wqkv[l], h->qkv, D, bn_of(rows, h->qkv))); h->tm_wqkv.push_back(m);
      FD_TRY(make_tmap_2d(&m, h->wo[l], D, size_t(H) * Dh, bn_of(rows, D, EPI_RESID, H * Dh)));
      h->tm_wo.push_back(m);
      if (h->fp8) {
        FD_TRY(make_tmap_2d_e4m3(&m, h->w1[l], h->dff, D, bn_of(rows, h->dff))); h->tm_w1.push_back(m);
        FD_TRY(make_tmap_2d_e4m3(&m, h->w2[l], D, h->dff, bn_of(rows, D, EPI_RESID, h->dff)));
        h->tm_w2.push_back(m);
      } else {
        FD_TRY(make_tmap_2d(&m, h->w1[l], h->dff, D, bn_of(rows, h->dff))); h->tm_w1.push_back(m);
        FD_TRY(make_tmap_2d(&m, h->w2[l], D, h->dff, bn_of(rows, D, EPI_RESID, h->dff)));
        h->tm_w2.push_back(m);
      }
    }
    const int n_out = h->paper ? c_px : h->c_out;
    FD_TRY(make_tmap_2d(&h->tm_wout, h->wout, n_out, D, bn_of(h->paper ? RM : L, n_out)));
    if (h->paper) {
      FD_TRY(make_tmap_2d(&h->tm_wup, h->wup, size_t(c.r_t) * D, D, bn_of(L, c.r_t * D)));
      FD_TRY(make_tmap_2d(&h->tm_wsp1, h->wsp1, D, D, bn_of(RM, D)));
      for (int tau = 0; tau < c.r_t; ++tau) {
        CUtensorMap m;
        FD_TRY(make_tmap_2d(&m, static_cast<char*>(h->xsb) + size_t(tau) * L * D * 2, L, D, 128));
        h->tm_xs.push_back(m);
      }
      if (h->ref_batch) FD_TRY(make_tmap_2d(&h->tm_xs_all, h->xsb, RM, D, 128));
      const uint64_t kd[3] = {64, uint64_t(h->rkv_rows), uint64_t(NR) * BG};
      const uint64_t ks[2] = {64 * 2, uint64_t(h->rkv_rows) * 64 * 2};
      const uint32_t kb[3] = {64, 64, 1};
      FD_TRY(make_tmap(&h->tm_rk, h->rkc, 3, kd, ks, kb));
      const uint64_t vd[3] = {uint64_t(h->rvt_pitch), 64, uint64_t(NR) * BG};
      const uint64_t vs[2] = {uint64_t(h->rvt_pitch) * 2, uint64_t(h->rvt_pitch) * 64 * 2};
      const uint32_t vb[3] = {64, 64, 1};
      FD_TRY(make_tmap(&h->tm_rv, h->rvtc, 3, vd, vs, vb));
    }
    {   // K [NB*G][kv_rows][64]: box 64 dims x 64 keys x 1
      const uint64_t dims[3] = {64, uint64_t(h->kv_rows), uint64_t(NB) * BG};
      const uint64_t str[2] = {64 * 2, uint64_t(h->kv_rows) * 64 * 2};
      const uint32_t box[3] = {64, 64, 1};
      FD_TRY(make_tmap(&h->tm_k, h->kc, 3, dims, str, box));
    }
    {   // V^T [NB*G][64][vt_pitch]: box 64 keys x 64 dims x 1
      const uint64_t dims[3] = {uint64_t(h->vt_pitch), 64, uint64_t(NB) * BG};
      const uint64_t str[2] = {uint64_t(h->vt_pitch) * 2, uint64_t(h->vt_pitch) * 64 * 2};
      const uint32_t box[3] = {64, 64, 1};
      FD_TRY(make_tmap(&h->tm_v, h->vtc, 3, dims, str, box));
    }
  }

  // ---- reset state, build the graph
  FD_CUDA(cudaMemset(h->kc, 0, h->k_bytes));
  FD_CUDA(cudaMemset(h->vtc, 0, h->v_bytes));
  if (h->paper) {
    FD_CUDA(cudaMemset(h->rkc, 0, h->rk_bytes));
    FD_CUDA(cudaMemset(h->rvtc, 0, h->rv_bytes));
  }
  FD_CUDA(cudaMemset(h->ctr, 0, size_t(h->B) * 8));
  FD_CUDA(cudaMemset(h->status, 0, 16));
  if (h->amax) FD_CUDA(cudaMemset(h->amax, 0, size_t(h->n_amax) * 4));
  FD_CUDA(cudaMemset(h->fs, 0, sizeof(FrameState)));
  FD_TRY(h->build_graph());
  FD_CUDA(cudaDeviceSynchronize());
  return FD_OK;
}

// Ordering between the caller's streams and the handle's host_stream (the
// graphs of fd_decode_frame_host run there). Every call that enqueues work on a
// caller stream first waits for the last such graph; fd_decode_frame_host first
// waits for the caller-stream work enqueued since the previous host call.
fd_status_t join_user_stream(fd_handle* h, cudaStream_t s) {
  if (h->g_last >= 0) {
    FD_CUDA(cudaStreamWaitEvent(s, h->ev_graph[h->g_last], 0));
    h->g_last = -1;
  }
  h->user_pending = true;
  h->last_stream = s;
  return FD_OK;
}

fd_status_t patch_io(fd_handle* h, const void* latent, void* out) {
  if (latent != h->cur_latent) {
    h->embed_p.latent = latent;
    void* args[] = {&h->embed_p};
    cudaKernelNodeParams np{};
    np.func = const_cast<void*>(h->embed_launch.func);
    np.gridDim = h->embed_launch.grid;
    np.blockDim = h->embed_launch.block;
    np.sharedMemBytes = unsigned(h->embed_launch.smem);
    np.kernelParams = args;
    FD_CUDA(cudaGraphExecKernelNodeSetParams(h->exec, h->embed_node, &np));
    h->cur_latent = latent;
  }
  if (out != h->cur_out) {
    for (OutNode& on : h->out_nodes) {
      on.p.out = out;
      cudaKernelNodeParams np{};
      np.func = const_cast<void*>(on.launch.func);
      np.gridDim = on.launch.grid;
      np.blockDim = on.launch.block;
      np.sharedMemBytes = unsigned(on.launch.smem);
      int K = on.K;
      if (h->bf) {
        CUtensorMap a = on.tmA, b = on.tmB;
        int* st = h->status;
        void* args[] = {&a, &b, &K, &on.p, &st};
        np.kernelParams = args;
        FD_CUDA(cudaGraphExecKernelNodeSetParams(h->exec, on.node, &np));
      } else {
        const float* a = static_cast<const float*>(on.A);
        const float* b = static_cast<const float*>(on.B);
        void* args[] = {&a, &b, &K, &on.p};
        np.kernelParams = args;
        FD_CUDA(cudaGraphExecKernelNodeSetParams(h->exec, on.node, &np));
      }
    }
    h->cur_out = out;
  }
  return FD_OK;
}

}  // namespace

extern "C" {

fd_status_t fd_create(const fd_config* cfg, const fd_weights* weights, fd_handle** out) {
  g_last_error.clear();
  if (out) *out = nullptr;
  if (!cfg || !weights || !out) return fail(FD_ERR_INVALID_ARG, "fd_create: null argument");
  FD_TRY(validate(cfg));
  const fd_weights* w = weights;
  if (!w->embed_w || !w->embed_b || !w->norm1_g || !w->wqkv || !w->bqkv || !w->wo || !w->bo ||
      !w->norm2_g || !w->w1 || !w->b1 || !w->w2 || !w->b2 || !w->final_g || !w->out_w ||
      !w->out_b || (cfg->kv_norm && (!w->knorm_g || !w->vnorm_g)) ||
      (cfg->head_mode == 1 && (!w->up_w || !w->up_b || !w->sp1_w || !w->sp1_b)))
    return fail(FD_ERR_INVALID_ARG, "fd_create: null weight pointer");
  const int n_all = cfg->n_blocks + (cfg->head_mode == 1 ? cfg->n_refine : 0);
  for (int l = 0; l < n_all; ++l)
    if (!w->norm1_g[l] || !w->wqkv[l] || !w->bqkv[l] || !w->wo[l] || !w->bo[l] ||
        !w->norm2_g[l] || !w->w1[l] || !w->b1[l] || !w->w2[l] || !w->b2[l] ||
        (cfg->kv_norm && (!w->knorm_g[l] || !w->vnorm_g[l])))
      return fail(FD_ERR_INVALID_ARG, "fd_create: null weight pointer in block %d", l);
  if (cfg->mlp_fp8) {
    if (!w->mlp_scales) return fail(FD_ERR_INVALID_ARG, "fd_create: mlp_fp8 needs mlp_scales");
    for (int l = 0; l < n_all; ++l) {
      const float* sc = w->mlp_scales[l];
      if (!sc || !(sc[0] > 0.f) || !(sc[1] > 0.f) || !std::isfinite(sc[0]) || !std::isfinite(sc[1]))
        return fail(FD_ERR_INVALID_ARG, "fd_create: FP8 scales of block %d must be finite and > 0", l);
    }
  }
  fd_handle* h = new (std::nothrow) fd_handle();
  if (!h) return fail(FD_ERR_OOM, "fd_create: host allocation failed");
  const fd_status_t s = create_impl(cfg, weights, h);
  if (s != FD_OK) {
    cudaDeviceSynchronize();
    cudaGetLastError();
    delete h;
    return s;
  }
  *out = h;
  return FD_OK;
}

fd_status_t fd_reset(fd_handle* h, void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_reset: invalid handle");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  FD_CUDA(cudaMemsetAsync(h->kc, 0, h->k_bytes, s));
  FD_CUDA(cudaMemsetAsync(h->vtc, 0, h->v_bytes, s));
  if (h->paper) {
    FD_CUDA(cudaMemsetAsync(h->rkc, 0, h->rk_bytes, s));
    FD_CUDA(cudaMemsetAsync(h->rvtc, 0, h->rv_bytes, s));
  }
  FD_CUDA(cudaMemsetAsync(h->ctr, 0, size_t(h->B) * 8, s));
  FD_CUDA(cudaMemsetAsync(h->status, 0, 16, s));
  if (h->amax) FD_CUDA(cudaMemsetAsync(h->amax, 0, size_t(h->n_amax) * 4, s));
  if (h->split_ctr) FD_CUDA(cudaMemsetAsync(h->split_ctr, 0, h->split_units_max * 4, s));
  h->last_stream = s;
  return FD_OK;
}

fd_status_t fd_reset_stream(fd_handle* h, int b, void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_reset_stream: invalid handle");
  if (b < 0 || b >= h->B) return fail(FD_ERR_INVALID_ARG, "fd_reset_stream: stream %d out of range", b);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  FD_CUDA(cudaMemsetAsync(h->ctr + b, 0, 8, s));
  h->last_stream = s;
  return FD_OK;
}

fd_status_t fd_stream_frame_index(fd_handle* h, int b, int64_t* t_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_stream_frame_index: invalid handle");
  if (b < 0 || b >= h->B || !t_out)
    return fail(FD_ERR_INVALID_ARG, "fd_stream_frame_index: bad stream or null output");
  FD_CUDA(cudaStreamSynchronize(h->last_stream));
  long long t = 0;
  FD_CUDA(cudaMemcpy(&t, h->ctr + b, 8, cudaMemcpyDeviceToHost));
  *t_out = t;
  return FD_OK;
}

fd_status_t fd_decode_frame(fd_handle* h, const void* latent, void* out, void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_decode_frame: invalid handle");
  if (!latent || !out) return fail(FD_ERR_INVALID_ARG, "fd_decode_frame: null buffer");
  if ((reinterpret_cast<uintptr_t>(latent) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(FD_ERR_INVALID_ARG, "fd_decode_frame: buffers must be 16-byte aligned");
  cudaPointerAttributes a{}, b{};
  FD_CUDA(cudaPointerGetAttributes(&a, latent));
  FD_CUDA(cudaPointerGetAttributes(&b, out));
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(FD_ERR_INVALID_ARG, "fd_decode_frame: latent_frame is not device memory");
  if (b.type != cudaMemoryTypeDevice && b.type != cudaMemoryTypeManaged)
    return fail(FD_ERR_INVALID_ARG, "fd_decode_frame: out_pixels is not device memory");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  FD_TRY(patch_io(h, latent, out));
  FD_CUDA(cudaGraphLaunch(h->exec, s));
  return FD_OK;
}

fd_status_t fd_decode_frame_host(fd_handle* h, const void* latent_host, void* out_host,
                                 void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_decode_frame_host: invalid handle");
  if (!latent_host || !out_host) return fail(FD_ERR_INVALID_ARG, "fd_decode_frame_host: null buffer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t g = h->host_stream;
  const int slot = h->host_slot;
  // the graph runs after the caller's earlier work (a reset, a device-buffer
  // decode) and after the copy-out that last read this slot's pixels
  if (h->user_pending) {
    FD_CUDA(cudaEventRecord(h->ev_user, h->last_stream));
    FD_CUDA(cudaStreamWaitEvent(g, h->ev_user, 0));
    h->user_pending = false;
  }
  if (h->d2h_pending[slot]) FD_CUDA(cudaStreamWaitEvent(g, h->ev_d2h[slot], 0));
  FD_CUDA(cudaMemcpyAsync(h->latent_stage[slot], latent_host, h->B * h->latent_elems * h->io_elt,
                          cudaMemcpyHostToDevice, g));
  FD_TRY(patch_io(h, h->latent_stage[slot], h->out_stage[slot]));
  FD_CUDA(cudaGraphLaunch(h->exec, g));
  FD_CUDA(cudaEventRecord(h->ev_graph[slot], g));
  // the copy-out on the caller's stream: synchronising it covers this frame,
  // while the next frame's graph can already run on host_stream
  FD_CUDA(cudaStreamWaitEvent(s, h->ev_graph[slot], 0));
  FD_CUDA(cudaMemcpyAsync(out_host, h->out_stage[slot], h->B * h->out_elems * h->io_elt,
                          cudaMemcpyDeviceToHost, s));
  FD_CUDA(cudaEventRecord(h->ev_d2h[slot], s));
  h->d2h_pending[slot] = true;
  h->g_last = slot;
  h->host_slot = slot ^ 1;
  h->last_stream = s;
  return FD_OK;
}

void fd_destroy(fd_handle* h) {
  if (!valid_handle(h)) return;
  cudaDeviceSynchronize();
  h->magic = kDead;
  delete h;
}

fd_status_t fd_status(fd_handle* h) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_status: invalid handle");
  FD_CUDA(cudaStreamSynchronize(h->last_stream));
  int st = 0;
  FD_CUDA(cudaMemcpy(&st, h->status, 4, cudaMemcpyDeviceToHost));
  if (st != 0) return fail(fd_status_t(st), "device reported status %d", st);
  return FD_OK;
}

const char* fd_error_string(fd_status_t s) {
  switch (s) {
    case FD_OK: return "ok";
    case FD_ERR_INVALID_ARG: return "invalid argument";
    case FD_ERR_UNSUPPORTED: return "unsupported configuration";
    case FD_ERR_OOM: return "out of device memory";
    case FD_ERR_CUDA: return "CUDA error";
    case FD_ERR_TIMEOUT: return "device-side wait timed out";
    case FD_ERR_BAD_HANDLE: return "invalid handle";
    case FD_ERR_BOUNDS: return "device-side bounds check failed (bounds-checked build)";
  }
  return "unknown status";
}

const char* fd_last_error(void) { return g_last_error.c_str(); }

fd_status_t fd_frame_index(fd_handle* h, int64_t* t_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_frame_index: invalid handle");
  if (!t_out) return fail(FD_ERR_INVALID_ARG, "fd_frame_index: null output");
  FD_CUDA(cudaStreamSynchronize(h->last_stream));
  long long t = 0;
  FD_CUDA(cudaMemcpy(&t, h->ctr, 8, cudaMemcpyDeviceToHost));
  *t_out = t;
  return FD_OK;
}

fd_status_t fd_device_bytes(fd_handle* h, size_t* bytes_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_device_bytes: invalid handle");
  if (!bytes_out) return fail(FD_ERR_INVALID_ARG, "fd_device_bytes: null output");
  *bytes_out = h->dev_bytes;
  return FD_OK;
}

fd_status_t fd_cache_bytes(fd_handle* h, size_t* bytes_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_cache_bytes: invalid handle");
  if (!bytes_out) return fail(FD_ERR_INVALID_ARG, "fd_cache_bytes: null output");
  *bytes_out = h->cache_bytes;
  return FD_OK;
}

fd_status_t fd_debug_read_slot(fd_handle* h, int block, int slot, int kv, float* host_dst) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_read_slot: invalid handle");
  const fd_config& c = h->cfg;
  if (block < 0 || block >= c.n_blocks || slot < 0 || slot > c.window || (kv != 0 && kv != 1) ||
      !host_dst)
    return fail(FD_ERR_INVALID_ARG, "fd_debug_read_slot: bad block/slot/kv/dst");
  FD_CUDA(cudaDeviceSynchronize());
  const int G = c.n_kv_heads, Dh = c.head_dim, L = h->L;
  const size_t n = size_t(G) * L * Dh;
  std::vector<uint8_t> raw;
  if (kv == 0) {
    raw.resize(n * h->elt);
    for (int g = 0; g < G; ++g) {
      const size_t src = ((size_t(block) * h->B * G + g) * h->kv_rows + size_t(slot) * L) * Dh * h->elt;
      FD_CUDA(cudaMemcpy(raw.data() + size_t(g) * L * Dh * h->elt,
                         static_cast<char*>(h->kc) + src, size_t(L) * Dh * h->elt,
                         cudaMemcpyDeviceToHost));
    }
    for (size_t i = 0; i < n; ++i)
      host_dst[i] = h->bf ? bf16_bits_to_f32(reinterpret_cast<uint16_t*>(raw.data())[i])
                          : reinterpret_cast<float*>(raw.data())[i];
  } else {
    // V^T [G][Dh][pitch] -> [G][L][Dh]
    std::vector<uint8_t> rows(size_t(L) * h->elt);
    for (int g = 0; g < G; ++g)
      for (int d = 0; d < Dh; ++d) {
        const size_t src = ((size_t(block) * h->B * G + g) * Dh + d) * h->vt_pitch + size_t(slot) * L;
        FD_CUDA(cudaMemcpy(rows.data(), static_cast<char*>(h->vtc) + src * h->elt,
                           size_t(L) * h->elt, cudaMemcpyDeviceToHost));
        for (int n2 = 0; n2 < L; ++n2)
          host_dst[(size_t(g) * L + n2) * Dh + d] =
              h->bf ? bf16_bits_to_f32(reinterpret_cast<uint16_t*>(rows.data())[n2])
                    : reinterpret_cast<float*>(rows.data())[n2];
      }
  }
  return FD_OK;
}

fd_status_t fd_debug_ring_layout(fd_handle* h, int block, int32_t* slots, int32_t* copies) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_ring_layout: invalid handle");
  const fd_config& c = h->cfg;
  const int n_all = c.n_blocks + (h->paper ? c.n_refine : 0);
  if (block < 0 || block >= n_all || !slots || !copies)
    return fail(FD_ERR_INVALID_ARG, "fd_debug_ring_layout: bad block or null output");
  const bool refine = h->paper && block >= c.n_blocks;
  *slots = refine ? h->ref_slots : c.window + 1;
  *copies = refine && h->ref_batch ? 2 : 1;
  return FD_OK;
}

fd_status_t fd_debug_read_ring(fd_handle* h, int block, int b, int slot, int kv, float* host_dst) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_read_ring: invalid handle");
  const fd_config& c = h->cfg;
  const bool refine = h->paper && block >= c.n_blocks;
  const int n_all = c.n_blocks + (h->paper ? c.n_refine : 0);
  // a mirrored refinement ring keeps slot s at s and s + ref_slots
  const int slots = refine ? h->ref_slots * (h->ref_batch ? 2 : 1) : c.window + 1;
  if (block < 0 || block >= n_all || b < 0 || b >= h->B || slot < 0 || slot >= slots ||
      (kv != 0 && kv != 1) || !host_dst)
    return fail(FD_ERR_INVALID_ARG, "fd_debug_read_ring: bad block/stream/slot/kv/dst");
  FD_CUDA(cudaDeviceSynchronize());
  const int G = c.n_kv_heads, Dh = c.head_dim, L = h->L;
  const int layer = refine ? block - c.n_blocks : block;
  const int rows = refine ? h->rkv_rows : h->kv_rows;
  const int pitch = refine ? h->rvt_pitch : h->vt_pitch;
  const char* kbase = static_cast<const char*>(refine ? h->rkc : h->kc);
  const char* vbase = static_cast<const char*>(refine ? h->rvtc : h->vtc);
  const size_t slab = (size_t(layer) * h->B + b) * G;      // first (layer, stream, group) slab
  const size_t n = size_t(G) * L * Dh;
  auto to_f32 = [&](const uint8_t* src, size_t i) {
    return h->bf ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(src)[i])
                 : reinterpret_cast<const float*>(src)[i];
  };
  if (kv == 0) {
    std::vector<uint8_t> raw(n * h->elt);
    for (int g = 0; g < G; ++g) {
      const size_t src = ((slab + g) * rows + size_t(slot) * L) * Dh * h->elt;
      FD_CUDA(cudaMemcpy(raw.data() + size_t(g) * L * Dh * h->elt, kbase + src,
                         size_t(L) * Dh * h->elt, cudaMemcpyDeviceToHost));
    }
    for (size_t i = 0; i < n; ++i) host_dst[i] = to_f32(raw.data(), i);
  } else {
    // V^T [G][Dh][pitch] -> [G][L][Dh]
    std::vector<uint8_t> rowbuf(size_t(L) * h->elt);
    for (int g = 0; g < G; ++g)
      for (int d = 0; d < Dh; ++d) {
        const size_t src = ((slab + g) * Dh + d) * pitch + size_t(slot) * L;
        FD_CUDA(cudaMemcpy(rowbuf.data(), vbase + src * h->elt, size_t(L) * h->elt,
                           cudaMemcpyDeviceToHost));
        for (int n2 = 0; n2 < L; ++n2)
          host_dst[(size_t(g) * L + n2) * Dh + d] = to_f32(rowbuf.data(), n2);
      }
  }
  return FD_OK;
}

fd_status_t fd_debug_set_frame_index(fd_handle* h, int b, int64_t t, void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_set_frame_index: invalid handle");
  if (b < 0 || b >= h->B || t < 0)
    return fail(FD_ERR_INVALID_ARG, "fd_debug_set_frame_index: bad stream or negative index");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  const long long v = t;
  FD_CUDA(cudaMemcpyAsync(h->ctr + b, &v, 8, cudaMemcpyHostToDevice, s));
  FD_CUDA(cudaStreamSynchronize(s));             // v lives on this stack frame
  h->last_stream = s;
  return FD_OK;
}

fd_status_t fd_debug_poison(fd_handle* h, int32_t what, void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_poison: invalid handle");
  if (what & ~int32_t(FD_POISON_RING | FD_POISON_SPLIT_COUNTERS))
    return fail(FD_ERR_INVALID_ARG, "fd_debug_poison: unknown flags 0x%x", unsigned(what));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  if (what & FD_POISON_RING) {
    // all-ones bytes: a NaN in both bf16 and fp32
    FD_CUDA(cudaMemsetAsync(h->kc, 0xFF, h->k_bytes, s));
    FD_CUDA(cudaMemsetAsync(h->vtc, 0xFF, h->v_bytes, s));
    if (h->paper) {
      FD_CUDA(cudaMemsetAsync(h->rkc, 0xFF, h->rk_bytes, s));
      FD_CUDA(cudaMemsetAsync(h->rvtc, 0xFF, h->rv_bytes, s));
    }
  }
  if ((what & FD_POISON_SPLIT_COUNTERS) && h->split_ctr)
    FD_CUDA(cudaMemsetAsync(h->split_ctr, 0x7F, h->split_units_max * 4, s));
  h->last_stream = s;
  return FD_OK;
}

fd_status_t fd_debug_block_mlp(fd_handle* h, int block, const float* x_host, float* out_host) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_debug_block_mlp: invalid handle");
  const fd_config& c = h->cfg;
  const int n_all = c.n_blocks + (h->paper ? c.n_refine : 0);
  if (block < 0 || block >= n_all || !x_host || !out_host)
    return fail(FD_ERR_INVALID_ARG, "fd_debug_block_mlp: bad block or null buffer");
  FD_CUDA(cudaDeviceSynchronize());
  // the block's own launch shape: a refinement block that runs all r_t
  // sub-frames at once gets r_t M rows (the caller's M first, zeros after),
  // so its kernels take the tile widths its weight maps were built for
  const bool ref = h->ref_batch && block >= c.n_blocks;
  const BlockIO io = ref ? h->refine_io(0) : h->backbone_io(0);
  const size_t n = size_t(h->M) * c.d_model;
  if (ref) FD_CUDA(cudaMemset(io.x32, 0, size_t(io.M) * c.d_model * 4));
  FD_CUDA(cudaMemcpy(io.x32, x_host, n * 4, cudaMemcpyHostToDevice));
  FD_CUDA(cudaMemset(h->o, 0, size_t(io.M) * c.n_heads * c.head_dim * h->elt));
  // a one-off graph of the block's post-attention kernels on the backbone
  // stream; no timing events, no calibration records
  cudaGraph_t saved_graph = h->graph;
  cudaGraphNode_t saved_last = h->last_node;
  const bool saved_is_kernel = h->last_is_kernel;
  const size_t saved_kinds = h->kinds.size();
  const int saved_timing = h->cfg.kernel_timing;
  unsigned* saved_amax = h->amax;
  cudaGraph_t g = nullptr;
  cudaGraphExec_t ex = nullptr;
  FD_CUDA(cudaGraphCreate(&g, 0));
  h->graph = g;
  h->last_node = nullptr;
  h->last_is_kernel = false;
  h->cfg.kernel_timing = 0;
  h->amax = nullptr;
  fd_status_t st = h->add_post_attention(block, io);
  h->graph = saved_graph;
  h->last_node = saved_last;
  h->last_is_kernel = saved_is_kernel;
  h->kinds.resize(saved_kinds);
  h->cfg.kernel_timing = saved_timing;
  h->amax = saved_amax;
  cudaError_t e = cudaSuccess;
  if (st == FD_OK) e = cudaGraphInstantiate(&ex, g, 0);
  if (st == FD_OK && e == cudaSuccess) e = cudaGraphLaunch(ex, nullptr);
  if (st == FD_OK && e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
  if (st == FD_OK && e == cudaSuccess)
    e = cudaMemcpy(out_host, io.x32, n * 4, cudaMemcpyDeviceToHost);
  if (ex) cudaGraphExecDestroy(ex);
  cudaGraphDestroy(g);
  if (st == FD_OK && e != cudaSuccess) {
    cudaGetLastError();
    st = fail(FD_ERR_CUDA, "fd_debug_block_mlp: %s", cudaGetErrorString(e));
  }
  return st;
}

}  // extern "C"

// Fixed device scratch of fd_decode_frame_static_scratch: the attention
// key-splitting counters and partials of one frame, for handles whose need
// fits (modest configurations). Layout, the same for every handle:
//   [0, kStaticCtrBytes)            split counters, one int per unit, cleared
//                                   by every call before its frame runs
//   [kStaticCtrBytes, ...)          partial O, then partial (max, sum)
// The counters never share bytes with another handle's partials, and the
// clearing makes each call independent of what an earlier call (or one that
// gave up on a timeout) left behind.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;
constexpr size_t kStaticCtrBytes = size_t(64) << 10;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
std::mutex g_static_mu;
void* g_static_base[64] = {};                 // per device, from cudaGetSymbolAddress
}  // namespace

extern "C" {

fd_status_t fd_decode_frame_static_scratch(fd_handle* h, const void* latent, void* out,
                                           void* stream) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_decode_frame_static_scratch: invalid handle");
  if (h->split_rows_max == 0 || h->attn_nodes.empty())   // this handle's attention uses no scratch
    return fd_decode_frame(h, latent, out, stream);
  // the largest attention launch shape with key splitting (one latent frame,
  // or all sub-frames of a batched refinement block)
  const size_t units = h->split_units_max;
  const size_t o_bytes = h->split_rows_max * 64 * 4;
  const size_t ml_bytes = h->split_rows_max * 2 * 4;
  const size_t need = kStaticCtrBytes + round_up(o_bytes, 256) + ml_bytes;
  if (units * 4 > kStaticCtrBytes || need > kStaticScratchBytes)
    return fail(FD_ERR_UNSUPPORTED,
                "fd_decode_frame_static_scratch: attention scratch of %zu bytes exceeds the fixed %zu",
                need, kStaticScratchBytes);
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev));
  if (dev != h->device)
    return fail(FD_ERR_INVALID_ARG,
                "fd_decode_frame_static_scratch: current device %d is not the handle's device %d",
                dev, h->device);
  if (dev < 0 || dev >= 64) return fail(FD_ERR_UNSUPPORTED, "fd_decode_frame_static_scratch: device %d", dev);
  char* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_base[dev]) FD_CUDA(cudaGetSymbolAddress(&g_static_base[dev], g_static_scratch));
    base = static_cast<char*>(g_static_base[dev]);
  }
  // point every attention node at the fixed scratch, replay, point them back
  // (a graph parameter update affects launches made after it only)
  auto set = [&](bool fixed) -> fd_status_t {
    for (AttnNode& an : h->attn_nodes) {
      TcAttnParams ap = an.p;
      if (fixed) {
        ap.counter = reinterpret_cast<int*>(base);
        ap.part_o = reinterpret_cast<float*>(base + kStaticCtrBytes);
        ap.part_ml = reinterpret_cast<float*>(base + kStaticCtrBytes + round_up(o_bytes, 256));
      }
      CUtensorMap a = an.tmQ, b = an.tmK, c = an.tmV;
      void* args[] = {&a, &b, &c, &ap};
      cudaKernelNodeParams np{};
      np.func = const_cast<void*>(an.launch.func);
      np.gridDim = an.launch.grid;
      np.blockDim = an.launch.block;
      np.sharedMemBytes = unsigned(an.launch.smem);
      np.kernelParams = args;
      FD_CUDA(cudaGraphExecKernelNodeSetParams(h->exec, an.node, &np));
    }
    return FD_OK;
  };
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  FD_TRY(join_user_stream(h, s));
  FD_CUDA(cudaMemsetAsync(base, 0, units * 4, s));
  const fd_status_t st_set = set(true);
  if (st_set != FD_OK) {
    const std::string msg = g_last_error;
    set(false);                        // never leave the graph on the shared array
    g_last_error = msg;
    return st_set;
  }
  const fd_status_t st = fd_decode_frame(h, latent, out, stream);
  const std::string msg = g_last_error;
  const fd_status_t back = set(false);
  if (st != FD_OK) {
    g_last_error = msg;
    return st;
  }
  return back;
}

fd_status_t fd_mlp_fp8_scales(fd_handle* h, float* scales_out, int32_t cap, int32_t* n_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_mlp_fp8_scales: invalid handle");
  if (!n_out) return fail(FD_ERR_INVALID_ARG, "fd_mlp_fp8_scales: null n_out");
  if (!h->amax)
    return fail(FD_ERR_INVALID_ARG, "fd_mlp_fp8_scales: handle created without record_mlp_amax");
  *n_out = h->n_amax;
  if (cap == 0) return FD_OK;
  if (!scales_out || cap < h->n_amax)
    return fail(FD_ERR_INVALID_ARG, "fd_mlp_fp8_scales: output array too small");
  FD_CUDA(cudaStreamSynchronize(h->last_stream));
  std::vector<unsigned> bits(h->n_amax);
  FD_CUDA(cudaMemcpy(bits.data(), h->amax, bits.size() * 4, cudaMemcpyDeviceToHost));
  for (int i = 0; i < h->n_amax; ++i) {
    float a;
    std::memcpy(&a, &bits[i], 4);
    scales_out[i] = a > 0.f ? float(double(a) / 448.0) : 1.f;
  }
  return FD_OK;
}

fd_status_t fd_selftest_wait_timeout(int32_t timeout_us) {
  g_last_error.clear();
  if (timeout_us < 1 || timeout_us > 10000000)
    return fail(FD_ERR_INVALID_ARG, "fd_selftest_wait_timeout: limit out of range");
  int* d_status = nullptr;
  FD_CUDA(cudaMalloc(&d_status, 4));
  fd_status_t result = FD_OK;
  int st = 0;
  cudaError_t e = cudaMemset(d_status, 0, 4);
  if (e == cudaSuccess) {
    wait_timeout_selftest_kernel<<<1, 32>>>(d_status, 1000ull * timeout_us);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&st, d_status, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(d_status, 0, 4);     // the context still works
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaFree(d_status);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FD_ERR_CUDA, "fd_selftest_wait_timeout: %s", cudaGetErrorString(e));
  }
  result = fd_status_t(st);
  if (result == FD_ERR_TIMEOUT) fail(FD_ERR_TIMEOUT, "device wait gave up after %d us as designed",
                                     timeout_us);
  return result;
}

fd_status_t fd_last_step_kernel_ms(fd_handle* h, float* ms_out, int32_t* kind_out, int32_t cap,
                                   int32_t* n_out) {
  if (!valid_handle(h)) return fail(FD_ERR_BAD_HANDLE, "fd_last_step_kernel_ms: invalid handle");
  if (!n_out) return fail(FD_ERR_INVALID_ARG, "fd_last_step_kernel_ms: null n_out");
  const int n = int(h->timed.size());
  *n_out = n;
  if (cap == 0) return FD_OK;
  if (!h->cfg.kernel_timing)
    return fail(FD_ERR_INVALID_ARG, "fd_last_step_kernel_ms: handle created with kernel_timing=0");
  if (!ms_out || !kind_out || cap < n)
    return fail(FD_ERR_INVALID_ARG, "fd_last_step_kernel_ms: output arrays too small");
  FD_CUDA(cudaEventSynchronize(h->events.back()));
  for (int i = 0; i < n; ++i) {
    float ms = 0.f;
    FD_CUDA(cudaEventElapsedTime(&ms, h->events[h->timed[i].begin], h->events[h->timed[i].end]));
    ms_out[i] = ms;
    kind_out[i] = h->timed[i].kind;
  }
  return FD_OK;
}

}  // extern "C"
