/*
 * flashdec.h — C ABI of the FlashDecoder streaming step on NVIDIA B200 (sm_100a).
 *
 * The operation. "FlashDecoder: Real-Time Latent-to-Pixel Streaming Decoder
 * with Transformers" (academ.us/article/2607.14898), Sec. 3.3 "Frame-by-Frame
 * Processing": a video's latent frames z_0 .. z_{T'-1} are decoded one at a
 * time. For frame t the latent is projected to L_frm tokens (Eq. 1); each
 * Transformer block computes new keys and values, appends them to a rolling
 * cache and evicts the oldest frame (Eq. 2), and the frame's queries attend,
 * with no mask, to every cached token. A final projection turns each token
 * into r_t pixel frames of P x P pixels (Sec. 3.4, Step 3). With head_mode 1
 * the output head is the paper's own (Sec. 3.4): a Linear D -> r_t D splits
 * each latent frame into r_t sub-frames (Eq. 3), refinement blocks stream
 * those sub-frames one after another with the same rolling-cache mechanism
 * (each sub-frame attends to the last r_t (W+1) sub-frames), and a 2-layer
 * MLP + PixelShuffle turns each refined sub-frame into one pixel frame.
 * With bf16 storage and L_frm a multiple of 8, all r_t sub-frames of a latent
 * frame pass each refinement block in one launch per kernel, each with its
 * own window of the ring (same results as one after another).
 *
 * Conventions of this library:
 *   - W (fd_config.window) counts PAST latent frames. The cache keeps the
 *     current frame plus W past frames, i.e. W+1 ring slots per block; frame t
 *     is stored in slot t mod (W+1). While t < W only the t+1 frames that
 *     exist are attended to (no padding).
 *   - Every call enqueues work on a CUDA stream and returns at once. A handle
 *     is not thread-safe; one handle decodes one video stream at a time.
 *   - All functions return FD_OK (0) or a negative fd_status_t. The message
 *     of the last failure on the calling thread is fd_last_error().
 *   - The library never falls back to another implementation: it runs its
 *     own sm_100a kernels or returns an error.
 */
#ifndef FLASHDEC_H
#define FLASHDEC_H

#include <stdint.h>
#include <stddef.h>

#if defined(__GNUC__)
#define FD_API __attribute__((visibility("default")))
#else
#define FD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fd_handle fd_handle;   /* opaque */

typedef enum {
  FD_OK = 0,
  FD_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, bad size, bad config */
  FD_ERR_UNSUPPORTED = -2,   /* valid config the kernels do not implement    */
  FD_ERR_OOM = -3,           /* device allocation failed                      */
  FD_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed             */
  FD_ERR_TIMEOUT = -5,       /* a device-side wait ran out (see fd_status)    */
  FD_ERR_BAD_HANDLE = -6,    /* null, destroyed or foreign handle             */
  FD_ERR_BOUNDS = -7         /* bounds-checked build only (libflashdec_debug.so):
                                a kernel computed a ring row, slot, V^T column,
                                split-partial index or pixel offset outside its
                                buffer, skipped that access and recorded this
                                code (see fd_status)                          */
} fd_status_t;

typedef enum { FD_F32 = 0, FD_BF16 = 1 } fd_dtype;

/* Decoder shape. Paper notation in brackets. */
typedef struct {
  int32_t latent_ch;     /* [C'] latent channels                                  */
  int32_t grid_h;        /* [H'] latent rows per frame                            */
  int32_t grid_w;        /* [W'] latent columns per frame                         */
  int32_t patch;         /* p in {1,2}: PixelUnshuffle of the latent (Sec. 4.3)   */
  int32_t d_model;       /* [D]                                                   */
  int32_t n_heads;       /* [N] query heads                                       */
  int32_t n_kv_heads;    /* [G] key/value groups (GQA); must divide n_heads       */
  int32_t head_dim;      /* [D_h]                                                 */
  int32_t n_blocks;      /* Transformer blocks                                    */
  int32_t mlp_ratio;     /* hidden width = mlp_ratio * D                          */
  int32_t window;        /* W: past latent frames kept (ring of W+1 slots)        */
  int32_t out_ch;        /* [C] pixel channels                                    */
  int32_t r_t;           /* [r_t] pixel frames per latent frame                   */
  int32_t px_per_token;  /* P: each token becomes a P x P pixel patch             */
  int32_t kv_norm;       /* 1: RMSNorm keys and values per head (Sec. 3.2)        */
  fd_dtype dtype;        /* FD_F32: fp32 throughout; FD_BF16: bf16 storage with
                            fp32 accumulation, fp32 residual stream and norms     */
  fd_dtype io_dtype;     /* element type of latent_frame and out_pixels           */
  float norm_eps;        /* RMSNorm epsilon (1e-6)                                */
  float rope_theta;      /* RoPE base (1e4)                                       */
  int32_t kernel_timing; /* CUDA events recorded inside the graph, read by
                            fd_last_step_kernel_ms: 0 off; 1 around every
                            kernel; 2 around each attention launch only (the
                            dominant kernel; negligible overhead)                */
  int32_t head_mode;     /* 0: final RMSNorm + Linear D -> C r_t P^2 + unpatchify.
                            1: the paper's head (Sec. 3.4): Linear D -> r_t D
                            (Eq. 3) into r_t sub-frames, streamed through
                            n_refine refinement blocks with a window of r_t (W+1)
                            sub-frames, then RMSNorm, Linear D -> D, GELU,
                            Linear D -> C P^2 and PixelShuffle per sub-frame    */
  int32_t n_refine;      /* refinement blocks (head_mode 1; 1 .. 8)              */
  int32_t mlp_fp8;       /* 1: every Transformer block's MLP (backbone and
                            refinement) multiplies FP8 E4M3 operands with static
                            per-tensor scales (Sec. 4.6, optimization 4). Needs
                            dtype BF16, d_model a multiple of 128 and
                            fd_weights.mlp_scales. Each MLP Linear multiplies
                            the E4M3 images of its own input and weight: W_1
                            and W_2 are quantized here, each with the scale
                            fp32(max|W| / 448), round to nearest even; the
                            first Linear's input RMSNorm(x) (gain included)
                            and the second's input GELU(..) with the static
                            scales of fd_weights.mlp_scales                */
  int32_t record_mlp_amax; /* 1 (mlp_fp8 = 0 only; d_model a multiple of 128):
                            record, per block, max |RMSNorm(x)| entering the
                            MLP and max |GELU output| since the last fd_reset;
                            read them as static scales with
                            fd_mlp_fp8_scales                               */
  int32_t batch;         /* B video streams decoded together (1 .. 64): every
                            call takes one latent frame of each stream; each
                            stream has its own frame counter and ring slots
                            ([FD] Eq. 1 carries a batch dimension B)          */
  int32_t attn_splits;   /* bf16 attention: split every (query tile, head)'s key
                            range over this many CTAs and combine the partial
                            results (1 .. 4); 0 = chosen from the launch's fit
                            to the GPU's CTA slots. Results differ from 1 only
                            by floating-point summation order.               */
  int32_t attn_issuer;   /* bf16 attention: which threads issue the tensor-core
                            products of a CTA. 1 = two threads (QK^T and PV
                            each wait for their own inputs), 2 = one thread
                            polling both; 0 = one thread for launches with at
                            least as many CTAs as the GPU has CTA slots and at
                            most 100 key tiles of 64 per CTA, two otherwise
                            (the faster of the two as measured). Results are
                            identical bit for bit.                           */
} fd_config;

/*
 * Weights: HOST float32 arrays in PyTorch Linear layout [out][in]. Per-block
 * entries are arrays of n_blocks pointers. fd_create copies everything; the
 * caller may free the arrays when it returns. For FD_BF16 the library folds
 * each RMSNorm gain into the Linear that follows it and rounds to bf16
 * (nearest even).
 *   embed_w [D][C' p^2], embed_b [D]                      (Eq. 1; channel
 *            order of a token = (c, dy, dx), tokens in raster order)
 *   norm1_g [D]; wqkv [(N+2G) D_h][D] rows ordered [Q heads | K heads |
 *            V heads], bqkv [(N+2G) D_h]; knorm_g, vnorm_g [D_h] (ignored
 *            when kv_norm = 0); wo [D][N D_h], bo [D]; norm2_g [D];
 *            w1 [mlp_ratio D][D], b1; w2 [D][mlp_ratio D], b2 [D]
 *   final_g [D]; out_w [C r_t P^2][D] with output channel order
 *            (c, tau, dy, dx); out_b [C r_t P^2]
 * With head_mode 1 the per-block arrays hold n_blocks + n_refine entries
 * (backbone blocks, then refinement blocks), final_g is the RMSNorm gain
 * before the spatial MLP, and:
 *   up_w [r_t D][D], up_b [r_t D]       temporal upsampling; output channels
 *            [tau D, (tau+1) D) form sub-frame tau
 *   sp1_w [D][D], sp1_b [D]             first spatial MLP layer
 *   out_w [C P^2][D], out_b [C P^2]     second layer, channel order (c, dy, dx)
 * (up_w .. sp1_b are ignored with head_mode 0.)
 * With mlp_fp8 = 1:
 *   mlp_scales[l] -> 2 floats {s_a, s_h}, one entry per block (backbone, then
 *            refinement): static scales of the inputs of the two MLP Linears,
 *            a = RMSNorm(x) (with gain norm2_g) and the GELU output h, stored
 *            as e4m3(a / s_a) and e4m3(h / s_h); rounding to nearest even,
 *            saturating at +-448. Ignored with mlp_fp8 = 0.
 */
typedef struct {
  const float *embed_w, *embed_b;
  const float *const *norm1_g, *const *wqkv, *const *bqkv;
  const float *const *knorm_g, *const *vnorm_g;
  const float *const *wo, *const *bo, *const *norm2_g;
  const float *const *w1, *const *b1, *const *w2, *const *b2;
  const float *final_g, *out_w, *out_b;
  const float *up_w, *up_b, *sp1_w, *sp1_b;
  const float *const *mlp_scales;
} fd_weights;

/*
 * Create a decoder on the current CUDA device: validates cfg, uploads the
 * weights, allocates the ring cache and all scratch once (nothing is
 * allocated per frame), builds the per-frame CUDA graph and leaves the
 * decoder reset (frame counter 0, cache zeroed). Synchronous.
 * Errors: FD_ERR_INVALID_ARG (null pointers, inconsistent shapes),
 * FD_ERR_UNSUPPORTED (e.g. head_dim not 32/64, patch not 1/2, bf16 with
 * D or widths not multiples of 64), FD_ERR_OOM, FD_ERR_CUDA. On error *out
 * is set to NULL and nothing is leaked.
 */
FD_API fd_status_t fd_create(const fd_config* cfg, const fd_weights* weights, fd_handle** out);

/*
 * Start a new video: frame counter := 0 and every ring slot zeroed, enqueued
 * on `stream` (a cudaStream_t; NULL = legacy default stream). Sec. 3.3: the
 * cache only ever holds frames of the current video. With batch > 1 this
 * resets every stream.
 */
FD_API fd_status_t fd_reset(fd_handle* h, void* stream);

/*
 * Start a new video in stream b (0 <= b < batch) only: its frame counter :=
 * 0, enqueued on `stream`; the other streams continue. Its ring slots are not
 * cleared: a stream at frame t only ever reads the slots of its frames
 * max(0, t-W) .. t, all written after the reset.
 */
FD_API fd_status_t fd_reset_stream(fd_handle* h, int b, void* stream);

/*
 * Decode the next latent frame ([FD] Sec. 3.3, steps (1)-(3), then the output
 * projection): enqueue one replay of the per-frame CUDA graph on `stream`.
 *   latent_frame: DEVICE pointer, [B][C'][H'][W'] contiguous, io_dtype: the
 *                 next frame of each of the B = batch streams.
 *   out_pixels:   DEVICE pointer, [B][C][r_t][H'P/p][W'P/p] contiguous, io_dtype.
 * Both are owned by the caller, must be 16-byte aligned and must stay valid
 * until the work on `stream` completes. Returns before the work finishes.
 * Frames must be fed strictly in order. Device-side failures are reported
 * by fd_status, not here.
 */
FD_API fd_status_t fd_decode_frame(fd_handle* h, const void* latent_frame, void* out_pixels,
                            void* stream);

/*
 * Same as fd_decode_frame with HOST buffers: copies the latent frame to the
 * device, decodes it and copies the pixels back. `out_pixels` is complete
 * once `stream` has been synchronised. The copy-out runs on `stream`; the
 * copy-in and the frame's graph run on a stream of the handle, after all work
 * enqueued on `stream` before this call and after the copy-out of two frames
 * earlier (two device staging slots, used in turn). So the copy-out of frame
 * t overlaps the decode of frame t+1 when the caller does not synchronise in
 * between. Results are bit-identical to fd_decode_frame. For truly
 * asynchronous copies both buffers should be pinned (cudaHostAlloc /
 * cudaHostRegister), and each out_pixels buffer must stay untouched until
 * its copy-out has completed.
 */
FD_API fd_status_t fd_decode_frame_host(fd_handle* h, const void* latent_frame_host,
                                 void* out_pixels_host, void* stream);

/* Free every device resource of the handle (synchronises the device first). */
FD_API void fd_destroy(fd_handle* h);

/*
 * Sticky device-side status of the handle: FD_OK, or FD_ERR_TIMEOUT if a
 * bounded wait inside a kernel ran out (the kernel then returned early and
 * its outputs are invalid). Synchronises the handle's last stream.
 */
FD_API fd_status_t fd_status(fd_handle* h);

/* Static description of a status code. */
FD_API const char* fd_error_string(fd_status_t s);

/* Message of the last failure on the calling thread ("" if none). */
FD_API const char* fd_last_error(void);

/* Number of frames decoded since the last reset (synchronises); stream 0. */
FD_API fd_status_t fd_frame_index(fd_handle* h, int64_t* t_out);

/* Same for stream b (0 <= b < batch). */
FD_API fd_status_t fd_stream_frame_index(fd_handle* h, int b, int64_t* t_out);

/* Device bytes held by the handle (weights, ring cache, scratch, staging). */
FD_API fd_status_t fd_device_bytes(fd_handle* h, size_t* bytes_out);

/* Bytes of the ring caches alone: n_blocks * 2 * G * (W+1) L_frm * D_h * elt,
 * plus, with head_mode 1, n_refine * 2 * G * S L_frm * D_h * elt where S is
 * the refinement ring's slots times their copies (fd_debug_ring_layout). */
FD_API fd_status_t fd_cache_bytes(fd_handle* h, size_t* bytes_out);

/*
 * Test/debug: copy ring slot `slot` of backbone block `block` of stream 0 to
 * host memory as fp32 [G][L_frm][D_h]. kv = 0 reads keys (stored after KV-norm and RoPE
 * at the frame's absolute index), kv = 1 reads values (after KV-norm).
 * Synchronous.
 */
FD_API fd_status_t fd_debug_read_slot(fd_handle* h, int block, int slot, int kv, float* host_dst);

/*
 * Test/debug: the ring layout of block `block` (as fd_debug_read_ring numbers
 * blocks): *slots = frames (or sub-frames) it holds, frame f in slot f mod
 * *slots; *copies = 1, or 2 when every slot is stored twice (slot s also at
 * s + *slots). The backbone has W+1 slots and one copy. The refinement ring
 * ([FD] Sec. 3.4 Step 2: each sub-frame attends to the last r_t (W+1)
 * sub-frames) has r_t (W+1) slots and one copy when sub-frames go through it
 * one at a time, and r_t (W+2) - 1 slots in two copies when all r_t
 * sub-frames of a latent frame go through it in one launch: writing them then
 * evicts no sub-frame an earlier one of the same frame still attends to, and
 * every window is one contiguous run of the doubled ring. This layout is the
 * library's own; the paper fixes only which sub-frames each one attends to.
 * Errors: FD_ERR_BAD_HANDLE, FD_ERR_INVALID_ARG (block out of range, null output).
 */
FD_API fd_status_t fd_debug_ring_layout(fd_handle* h, int32_t block, int32_t* slots,
                                        int32_t* copies);

/*
 * Test/debug: copy ring slot `slot` of block `block`, video stream b
 * (0 <= b < batch), to host memory as fp32 [G][L_frm][D_h]. Blocks
 * 0 .. n_blocks-1 are the backbone (slots 0 .. W); with head_mode 1, blocks
 * n_blocks .. n_blocks + n_refine - 1 are the refinement blocks, whose slots
 * and copies fd_debug_ring_layout gives (slot < slots x copies; slot
 * s + slots is the second copy of slot s). kv as for fd_debug_read_slot.
 * Synchronous.
 */
FD_API fd_status_t fd_debug_read_ring(fd_handle* h, int block, int b, int slot, int kv,
                                      float* host_dst);

/*
 * Test/debug: fill device state with values that must never reach an output,
 * enqueued on `stream`. FD_POISON_RING sets every byte of the ring caches
 * (backbone and refinement) to 0xFF, a NaN in bf16 and fp32: a decode after
 * fd_reset + this call must give the same outputs as after fd_reset alone,
 * because a frame only reads ring slots written since the reset ([FD] Sec. 3.3:
 * the cache holds only frames that exist). FD_POISON_SPLIT_COUNTERS sets the
 * attention key-splitting counters to 0x7F7F7F7F, which breaks the handle's own
 * split combine until the next fd_reset (a positive control for the fixed-
 * scratch entry point below).
 */
enum { FD_POISON_RING = 1, FD_POISON_SPLIT_COUNTERS = 2 };
FD_API fd_status_t fd_debug_poison(fd_handle* h, int32_t what, void* stream);

/*
 * Test/debug: set stream b's frame counter to t (>= 0), so that the next
 * decoded frame is treated as frame t (ring slot t mod (W+1), temporal RoPE
 * at index t); nothing else changes. Lets a test reach very long videos
 * ([FD] Sec. 4.3 "Long Video Decoding": length is unbounded) without decoding
 * every frame before them: once n_blocks W + 1 frames have been decoded after
 * the jump, every slot that frame t reads was written after it, so the output
 * equals that of a video that really started at frame 0 (positions enter the
 * attention only through differences). Synchronous on `stream`.
 */
FD_API fd_status_t fd_debug_set_frame_index(fd_handle* h, int b, int64_t t, void* stream);

/*
 * Test/debug: run the second half of block `block` (backbone blocks first,
 * then refinement blocks) once on a given residual stream: x_host becomes
 * the stream, the attention output is set to zero, and the
 * block's O-projection (so x + b_o), MLP-up and MLP-down kernels (with
 * mlp_fp8 the E4M3 quantization of RMSNorm(x + b_o) in between) run with the
 * handle's weights; the resulting stream x + b_o + MLP(x + b_o) is copied to
 * out_host. Both are [batch L_frm][D] fp32. Both sides of a parity test then
 * start the MLP from identical float32 values. Synchronous;
 * overwrites the handle's per-frame scratch (not the ring cache), so it must
 * not overlap a decode; records no calibration ranges.
 */
FD_API fd_status_t fd_debug_block_mlp(fd_handle* h, int block, const float* x_host,
                                      float* out_host);

/*
 * Kernel timing (requires cfg.kernel_timing = 1 or 2): waits for the last
 * enqueued frame and writes the device time in ms of each timed kernel of
 * that frame (every kernel, or every attention launch), in launch order, to
 * ms_out[0 .. n-1] and its kind to kind_out (see fd_kernel_kind).
 * *n_out = number of timed kernels per frame. Pass cap = 0 to query *n_out
 * only. Each replay of the frame graph overwrites the previous frame's times.
 */
/* With head_mode 1 a frame runs, after the backbone: UPSAMPLE once, then the
 * refinement blocks' QKV .. MLP_DOWN kernels, SPATIAL (first MLP layer) and
 * FINAL (second layer + PixelShuffle): once over all r_t sub-frames when the
 * refinement ring has two copies (fd_debug_ring_layout), else per sub-frame. */
typedef enum {
  FD_K_STEP_BEGIN = 0, FD_K_EMBED = 1, FD_K_QKV = 2, FD_K_ATTN = 3,
  FD_K_OPROJ = 4, FD_K_MLP_UP = 5, FD_K_MLP_DOWN = 6, FD_K_FINAL = 7,
  FD_K_UPSAMPLE = 8, FD_K_SPATIAL = 9,
  FD_K_MLP_NORM = 10   /* mlp_fp8: RMSNorm + E4M3 quantization of the MLP input
                          (after each O-projection); record_mlp_amax: its range */
} fd_kernel_kind;
FD_API fd_status_t fd_last_step_kernel_ms(fd_handle* h, float* ms_out, int32_t* kind_out,
                                   int32_t cap, int32_t* n_out);

/*
 * fd_decode_frame without the handle's attention scratch (the paper has no
 * counterpart: this is a deployment variant of this library). Identical
 * results to fd_decode_frame. Some callers cannot allocate device memory at
 * the point where they decode: code running inside a host that pre-plans all
 * of its memory (an inference server's memory pool or a pre-allocated arena),
 * or that must not call cudaMalloc between two frames because it would
 * synchronise the device and break a frame's latency budget. When the
 * handle's attention splits its key ranges (fd_config.attn_splits, or the
 * automatic choice), the partial results and counters of that split live in
 * one fixed, statically sized device array of this library (8 MiB) instead of
 * memory allocated by fd_create; this call allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine). Handles whose split needs more
 * than the array (64 KiB of counters, then (L/128 rounded up) x heads x batch
 * x splits x 33 KB of partials) get FD_ERR_UNSUPPORTED; handles that do not
 * split simply run fd_decode_frame.
 *  - The array is shared by every handle and stream of the process on that
 *    device and keeps the last call's contents. Each call first clears the
 *    counters it uses (an enqueued memset, no allocation), so serialised calls
 *    of different handles are independent. Calls that overlap in time
 *    (different streams, threads or handles, or an
 *    fd_decode_frame_static_scratch still running on the GPU when another is
 *    enqueued on a different stream) race on it and give wrong results.
 *    Serialise them on one stream.
 *  - The current device must be the one the handle was created on
 *    (FD_ERR_INVALID_ARG otherwise). The first call on each device resolves
 *    the array's address there (cudaGetSymbolAddress); make that first call
 *    outside any CUDA stream capture. Each call also updates the attention
 *    nodes of the handle's frame graph before and after enqueueing it, and
 *    puts them back on the handle's own scratch even when it fails.
 * Errors as for fd_decode_frame, plus FD_ERR_UNSUPPORTED for oversize.
 */
FD_API fd_status_t fd_decode_frame_static_scratch(fd_handle* h, const void* latent_frame,
                                                  void* out_pixels, void* stream);

/*
 * Static FP8 scales from the calibration recorded by a handle created with
 * record_mlp_amax = 1 ([FD] Sec. 4.6: static calibration): for every block
 * (backbone, then refinement), scales_out[2 l] = fp32(max |RMSNorm(x)| / 448) and
 * scales_out[2 l + 1] = fp32(max |h| / 448) over the frames decoded since the
 * last fd_reset (1 where nothing was seen), ready for fd_weights.mlp_scales of
 * an mlp_fp8 handle. *n_out = 2 * (n_blocks + n_refine); cap = 0 queries it.
 * Synchronises the handle's last stream. FD_ERR_INVALID_ARG if the handle
 * does not record.
 */
FD_API fd_status_t fd_mlp_fp8_scales(fd_handle* h, float* scales_out, int32_t cap,
                                     int32_t* n_out);

/*
 * Self-test of the device-side failure path (no handle needed; runs on the
 * current device and synchronises it). Every device wait of the decoder's
 * kernels is bounded; this launches one tiny kernel that waits, with the same
 * bounded-wait code and a limit of timeout_us microseconds (1 .. 10^7), on an
 * mbarrier that nothing ever completes. Returns FD_ERR_TIMEOUT when the wait
 * gave up as designed and the GPU context is still usable afterwards, FD_OK
 * if the wait wrongly succeeded, FD_ERR_INVALID_ARG for a bad limit and
 * FD_ERR_CUDA for a runtime failure. No fault, trap or hang is involved.
 */
FD_API fd_status_t fd_selftest_wait_timeout(int32_t timeout_us);

#ifdef __cplusplus
}
#endif
#endif /* FLASHDEC_H */
