/*
 * bv.h -- C ABI of the B200 BigVGAN alias-free waveform decoder (libbv.so).
 *
 * The operations follow the BigVGAN-style decoders described on
 *   [H3]  docs.rs cortiq-engine 0.5.74, src/cortiq_engine/audiovae.rs
 *         (MiniMax-H3 audio VAE decoder, 32 kHz)
 *   [LTX] docs.rs cortiq-engine 0.6.3, src/cortiq_engine/ltxaudio.rs
 *         (LTX-2.5 BigVGAN v2 vocoder, 16 kHz)
 *   [M3]  docs.rs cortiq-engine 0.5.89, src/cortiq_engine/music3.rs
 *         (overlapping windows averaged by coverage, used for tiling)
 *
 * Conventions for every call:
 *  - Tensors are contiguous float32 [B, C, T] (T fastest).  Stereo is B = 2
 *    independent mono passes, as both decoders run it.
 *  - Every tensor pointer is a caller-owned DEVICE pointer unless the
 *    argument says host.  The library never allocates, frees or keeps device
 *    memory between calls; scratch lives in the caller's workspace.  Pointers
 *    must be 4-byte aligned; workspaces 256-byte aligned.
 *  - Calls enqueue work on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and return without synchronising.  They perform no allocation,
 *    no synchronisation and no host<->device copy, so they may be captured
 *    into a CUDA graph, after a first uncaptured call on the device (which
 *    sets kernel attributes).
 *  - Errors are returned, never aborted on: argument and shape errors are
 *    detected before anything is launched and leave the outputs untouched;
 *    launch failures return BV_ERR_CUDA.  bv_last_error() gives a message for
 *    the calling thread's last failing call.
 *  - There is no CPU fallback: without a usable sm_100 device every compute
 *    call returns BV_ERR_CUDA.
 */
#ifndef BV_H_
#define BV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BV_OK = 0,
  BV_ERR_ARG = 1,         /* null/misaligned/overlapping pointer, bad scalar */
  BV_ERR_SHAPE = 2,       /* inconsistent or out-of-range sizes */
  BV_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  BV_ERR_CUDA = 4,        /* a CUDA call failed (message has the CUDA error) */
  BV_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
  BV_ERR_UNSUPPORTED = 6, /* a valid request this build does not implement */
  BV_ERR_RANGE = 7        /* an activation reached fp16's range (|v| >= 65504),
                             or a weight 16 or more (2^12 |w| >= 65504), on the
                             fp16 time-major path; that output is not valid */
} bv_status;

#define BV_FILTER_TAPS 12 /* both resampling filters: 12 taps ([H3] FILTER_LEN) */
#define BV_MAX_UP 8       /* transposed-conv stages */
#define BV_MAX_BLOCKS 4   /* AMP blocks per stage */
#define BV_MAX_DIL 4      /* residual units (dilations) per AMP block */

/* Message for the calling thread's last failing call ("" if none). */
const char *bv_last_error(void);

/* Library version string. */
const char *bv_version(void);

/* Number of kernels this process has launched through the library. */
uint64_t bv_launch_count(void);

/* Per-kernel timing ([H3] `AVAE_TIME` phase timers, rebuilt on the device):
 * while enabled, every kernel the library launches is bracketed by a pair of
 * CUDA events on its stream and tagged with its kernel class and its
 * algorithmic FLOPs and bytes.  Enabling it creates events (host-side
 * resources) and adds two event records per launch; leave it off for
 * production and for CUDA-graph capture. */
typedef struct {
  char name[32];      /* kernel class: activation, conv1d, conv_transpose1d, tiles */
  uint64_t launches;
  double ms;          /* summed event time of the class's launches */
  double flops;       /* summed algorithmic FLOPs (2 per multiply-add) */
  double bytes;       /* summed algorithmic HBM bytes (each operand once) */
} bv_kernel_stats;

void bv_timing_enable(int on);
/* Synchronises the recorded events and writes up to `max` classes into
 * `out`; returns the number of classes (or -1 on a CUDA error).  The records
 * are kept until bv_timing_reset(). */
int bv_timing_read(bv_kernel_stats *out, int max);
void bv_timing_reset(void);

/* Reads and clears the device status word that bounded device-side waits
 * set when they give up, and that the activation feeding the fp16 time-major
 * convs sets when a value reaches |v| >= 65504 (fp16's range: the convs of
 * channel counts that are multiples of 8 from 48 up take their operands in
 * two fp16 parts); returns BV_OK, BV_ERR_TIMEOUT or BV_ERR_RANGE.
 * Synchronises `stream`. */
bv_status bv_sync_status(void *stream);

/* Testing hook for the bounded waits.  The tensor-core kernels poll each
 * mbarrier at most `polls` times (default 2^26) before they give up: the
 * CTA (and its pair) then stops issuing work, lets the copies and MMAs it
 * issued finish (each with its own fixed bound), frees its tensor memory,
 * sets the status word that bv_sync_status reads, and leaves its output
 * tile unspecified.  polls < 0 restores the default.  Takes effect for
 * launches enqueued after the call, process-wide; returns the previous
 * value.  A limit low enough to expire in a normal launch is for tests of
 * that unwinding only. */
long long bv_debug_set_wait_limit(long long polls);

/* ------------------------------------------------------------------------
 * Kaiser-windowed sinc lowpass design, on the host.
 * [H3] `kaiser_sinc(cutoff, half_width, k)` and `bessel_i0`, `sinc`:
 *   A = 2.285 (k/2 - 1) pi (4 half_width) + 7.95,
 *   beta = 0.1102 (A - 8.7) if A > 50; 0.5842 (A-21)^0.4 + 0.07886 (A-21) if
 *   21 <= A <= 50; else 0,
 *   w_i = I0(beta sqrt(1 - r_i^2)) / I0(beta), r_i = 2 i / (k - 1) - 1,
 *   f_i = 2 cutoff w_i sinc(2 cutoff (i - k/2 + 1/2)) (even k; odd k centres
 *   on i - k/2), normalised to unit sum, computed in double and rounded to
 *   float.  The decoders use (0.25, 0.3, 12) for both filters.
 * out_host: `taps` floats of HOST memory.  Errors: BV_ERR_ARG for a null
 * pointer, taps outside [1, 64], cutoff outside (0, 0.5] or half_width <= 0.
 * ---------------------------------------------------------------------- */
bv_status bv_filter_design(double cutoff, double half_width, int taps,
                           float *out_host);

/* ------------------------------------------------------------------------
 * Alias-free activation over x, y [B, C, T]:  y = down(snake(up(x))).
 * [H3] `Activation1d::apply`, `SnakeBeta`, `fir_pad`; [LTX] `Aliasing`,
 * `SnakeBeta::forward`.  Per row (b, c) of length n = T:
 *   up:    u[m] = 2 sum_j f_up[j] x[clamp((m + 15 - j)/2 - 5, 0, n-1)] over
 *          j with m + 15 - j even, m in [0, 2n)  (replicate pad 5, stride-2
 *          transposed FIR with gain 2, trim 15 each side);
 *   snake: v[m] = u[m] + sin^2(e^{log_alpha[c]} u[m]) / (e^{log_beta[c]} + eps);
 *   down:  y[t] = sum_{j<12} f_down[j] v[clamp(2t + j - 5, 0, 2n-1)].
 * The 2x signal never leaves the chip.  log_alpha, log_beta: [C] device;
 * up_filter, down_filter: [12] device.  x and y must not overlap (no
 * in-place).  eps is 1e-9 in both decoders.  Errors: BV_ERR_ARG (null or
 * overlapping pointers), BV_ERR_SHAPE (B, C, T < 1, or B*C*T >= 2^40).
 * ---------------------------------------------------------------------- */
bv_status bv_activation1d(const float *x, float *y, int B, int C, int T,
                          const float *log_alpha, const float *log_beta,
                          const float *up_filter, const float *down_filter,
                          float eps, void *stream);

/* The scalar sin^2 of the activation kernel, elementwise on n device floats
 * (out may equal z): exposed so its accuracy can be tested.  The activation
 * takes it for arguments past its fast path (|a u| > 51472; the fast path
 * works in units of pi with a degree-4 polynomial and is covered by the
 * activation's parity tests).  Method: additive reduction by pi (sin^2 has
 * period pi) with pi split in three floats (Cody & Waite), then the Taylor
 * series of sin to r^13 on |r| <= pi/2, squared; |z| > 65536 uses sinf. */
bv_status bv_sin_squared(const float *z, float *out, int64_t n, void *stream);

/* Epilogue fused into the convolutions.  With v = conv(x) + bias:
 *   v = scale * (v + residual);  if accumulate: v += y (previous contents);
 *   v = final_act(v);  y = v.
 * residual: [B, Cout, Tout] device or NULL; it may be y itself (in-place
 * residual update) but must not partially overlap y.  final_act: 0 none,
 * 1 clamp to [-1, 1] ([H3] decode, [LTX] apply_final), 2 tanh.
 * [H3] `AmpBlock::apply` (cur += conv), `AudioVae::decode` (stage mean,
 * clamp); [LTX] `AmpBlock::forward`, `Vocoder::forward`. */
typedef struct {
  const float *residual;
  float scale;
  int accumulate;
  int final_act;
} bv_epilogue;

/* ------------------------------------------------------------------------
 * Dilated Conv1d with zero padding ([H3] `Conv1d::apply`, [LTX]
 * `Conv1d::forward`):
 *   y[b,o,t] = bias[o] + sum_{i<Cin} sum_{j<K} w[o,i,j] x[b,i,t + j*dilation - pad],
 *   Tout = T + 2 pad - dilation (K - 1) >= 1.
 * x [B, Cin, T]; w [Cout, Cin, K] (PyTorch layout); bias [Cout] or NULL;
 * ep NULL = plain conv; y [B, Cout, Tout].  x must not overlap y.
 * Errors: BV_ERR_ARG, BV_ERR_SHAPE (sizes < 1, Tout < 1, K > 32).
 * ---------------------------------------------------------------------- */
bv_status bv_conv1d(const float *x, int B, int Cin, int T, const float *w,
                    const float *bias, int Cout, int K, int dilation, int pad,
                    const bv_epilogue *ep, float *y, void *stream);

/* ------------------------------------------------------------------------
 * ConvTranspose1d ([H3] `ConvT1d::apply`, [LTX] `ConvT1d::forward`): the
 * scatter  y[b, o, t*stride + j - pad] += x[b, i, t] w[i, o, j]  plus bias[o],
 * computed as the equivalent gather per output phase, so no atomics:
 *   y[b,o,p] = bias[o] + sum_i sum_{j = (p+pad) mod s + s m < K}
 *              x[b, i, (p + pad - j)/s] w[i, o, j]  (terms with the input
 *              index in [0, T)),
 *   Tout = (T - 1) stride + K - 2 pad >= 1.
 * x [B, Cin, T]; w [Cin, Cout, K] (PyTorch layout); bias [Cout] or NULL;
 * y [B, Cout, Tout].  x must not overlap y.  The decoders use K = 2 stride,
 * pad = (K - stride) / 2.  Errors: BV_ERR_ARG, BV_ERR_SHAPE (sizes < 1,
 * stride > 16, K > 64, Tout < 1).
 * ---------------------------------------------------------------------- */
bv_status bv_conv_transpose1d(const float *x, int B, int Cin, int T,
                              const float *w, const float *bias, int Cout,
                              int K, int stride, int pad, float *y,
                              void *stream);

/* ------------------------------------------------------------------------
 * One activation followed by one Conv1d -- the unit step of an AMP block
 * ([H3] `AmpBlock::apply`: `Activation1d::apply` then `Conv1d::apply`;
 * [LTX] `AmpBlock::forward`) -- on the kernels the decoder itself runs:
 *   h = down(snake(up(x)))            (as bv_activation1d, C channels)
 *   y = epilogue(conv(h; w, bias, K, dilation, pad))   (as bv_conv1d)
 * x [B, C, T]; log_alpha, log_beta [C]; filters [12]; w [Cout, C, K];
 * bias [Cout] or NULL; y [B, Cout, T + 2 pad - dilation (K - 1)]; all
 * device.  When the conv qualifies for the time-major tensor-core path
 * (C a multiple of 4 with at most a third of channel padding to 32-channel
 * blocks, Cout >= 40 or Cout = 32 with C a multiple of 32, (K - 1) dilation
 * <= 56) the activation's output is laid out time-major and the conv runs
 * there, as inside bv_decode: in two fp16 parts where C is a multiple of 8
 * from 48 up (activations below 65504 in magnitude, else bv_sync_status
 * reports BV_ERR_RANGE; see bv_decoder_config.tf32_only), else in 3xTF32.
 * Workspace: bv_act_conv1d_workspace_size bytes, 256-byte aligned, disjoint
 * from x, y and the residual.  x must not overlap y; the residual may be y.
 * Errors: BV_ERR_ARG, BV_ERR_SHAPE (sizes < 1, K > 32, output length < 1),
 * BV_ERR_WORKSPACE.
 * ---------------------------------------------------------------------- */
size_t bv_act_conv1d_workspace_size(int B, int C, int T, int Cout, int K,
                                    int dilation);
bv_status bv_act_conv1d(const float *x, int B, int C, int T,
                        const float *log_alpha, const float *log_beta,
                        const float *up_filter, const float *down_filter,
                        float eps, const float *w, const float *bias, int Cout,
                        int K, int dilation, int pad, const bv_epilogue *ep,
                        float *y, void *workspace, size_t ws_bytes,
                        void *stream);

/* bv_conv_transpose1d on the kernels the decoder runs for its upsampling
 * stages: with the workspace the phases run on the time-major tensor-core
 * kernel (or the [B, C, T] one) where the shape qualifies, else on the FP32
 * kernel (then the workspace may be empty).  The time-major kernel takes the
 * fp16 split where Cin is a multiple of 8 from 48 up, as bv_act_conv1d
 * (inputs below 65504 in magnitude), else 3xTF32.  Arguments, result and errors
 * as bv_conv_transpose1d, plus BV_ERR_WORKSPACE.  Workspace:
 * bv_conv_transpose1d_workspace_size bytes, 256-byte aligned, disjoint
 * from x and y. */
size_t bv_conv_transpose1d_workspace_size(int B, int Cin, int T, int Cout,
                                          int K, int stride);
bv_status bv_conv_transpose1d_ws(const float *x, int B, int Cin, int T,
                                 const float *w, const float *bias, int Cout,
                                 int K, int stride, int pad, float *y,
                                 void *workspace, size_t ws_bytes,
                                 void *stream);

/* ------------------------------------------------------------------------
 * One AMP (anti-aliased multi-periodicity) residual block, [H3]
 * `AmpBlock::apply`, [LTX] `AmpBlock::forward`: the units run in sequence,
 *   cur = x;  for u < n_dilations:
 *     h = act(cur; act_log_alpha/beta[2u]);
 *     h = conv(h; conv1 w/b[u], K, dilation[u], pad (K d - d)/2);
 *     h = act(h; act_log_alpha/beta[2u+1]);
 *     h = conv(h; conv2 w/b[u], K, 1, pad (K-1)/2);
 *     cur = cur + h;
 * and the result is written as  y = (accumulate ? y : 0) + scale * cur
 * (the decoder averages a stage's blocks with scale = 1/n_blocks).
 * All weights are device pointers in PyTorch layout ([C, C, K], biases [C]
 * or NULL, log_alpha/log_beta [C], filters [12]).
 * ---------------------------------------------------------------------- */
typedef struct {
  int kernel_size;            /* odd K of every conv in the block */
  int n_dilations;            /* 1..BV_MAX_DIL */
  int dilation[BV_MAX_DIL];
  const float *conv1_w[BV_MAX_DIL];
  const float *conv1_b[BV_MAX_DIL];
  const float *conv2_w[BV_MAX_DIL];
  const float *conv2_b[BV_MAX_DIL];
  const float *act_log_alpha[2 * BV_MAX_DIL];
  const float *act_log_beta[2 * BV_MAX_DIL];
  const float *up_filter;     /* [12] */
  const float *down_filter;   /* [12] */
} bv_amp_params;

/* Workspace bytes bv_amp_block needs for [B, C, T]. */
size_t bv_amp_block_workspace_size(int B, int C, int T);

/* Workspace bytes with which bv_amp_block runs the block's convs on the
 * tensor cores from time-major operands (the path bv_decode takes): room for
 * two [B, T, C] operand planes and the convs' weights split into hi / lo
 * parts (fp16 where C is a multiple of 8 from 48 up, as bv_act_conv1d; else
 * tf32), besides the three [B, C, T] buffers.  Equals
 * bv_amp_block_workspace_size when no conv of the block qualifies (narrow
 * channel counts, or no tensor-core support); 0 for invalid arguments. */
size_t bv_amp_block_workspace_size_tc(int B, int C, int T, const bv_amp_params *p);

/* x, y [B, C, T] must not overlap each other or the workspace.  With a
 * workspace of at least bv_amp_block_workspace_size_tc bytes the qualifying
 * convs run time-major on the tensor cores; with at least
 * bv_amp_block_workspace_size bytes all convs read [B, C, T] operands.
 * Errors: BV_ERR_ARG, BV_ERR_SHAPE, BV_ERR_WORKSPACE. */
bv_status bv_amp_block(const float *x, int B, int C, int T,
                       const bv_amp_params *p, float *y, float scale,
                       int accumulate, void *workspace, size_t ws_bytes,
                       void *stream);

/* ------------------------------------------------------------------------
 * bv_amp_block without a workspace argument.  The pages have no counterpart
 * to this entry point: it exists for callers that cannot allocate device
 * memory when they run the block -- a real-time audio thread (a plugin's
 * render callback must not call cudaMalloc, which may block on the driver),
 * or a host that fixes its device memory budget before the decoder runs.
 * The scratch lives in a static device array inside libbv, sized for
 * B*C*T <= BV_AMP_STATIC_MAX_ELEMS (three tensors of that many floats,
 * 12 MiB); every GPU that loads the library holds it until the process
 * exits.  Larger requests return BV_ERR_WORKSPACE and leave y untouched.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture begins.  All calls share the one array and it
 * keeps the last call's contents (nothing in it needs to start at zero):
 * calls whose GPU work can overlap -- on different streams or from
 * different host threads -- race on it, so serialise them.  Arguments and
 * results are those of bv_amp_block.
 * ---------------------------------------------------------------------- */
#define BV_AMP_STATIC_MAX_ELEMS (1 << 20)

bv_status bv_amp_block_static(const float *x, int B, int C, int T,
                              const bv_amp_params *p, float *y, float scale,
                              int accumulate, void *stream);

/* ------------------------------------------------------------------------
 * The whole decoder ([H3] `AudioVae::decode`, [LTX] `Vocoder::forward`):
 *   conv_pre (pad (pre_kernel-1)/2)
 *   -> for each stage i: ConvT (rate up_rate[i], kernel up_kernel[i],
 *      pad (k - s)/2, channels -> up_channels[i]), then the mean of the
 *      stage's n_blocks AMP blocks (kernel block_kernel[j], the shared
 *      dilations), each fed the ConvT output
 *   -> act_post -> conv_post (pad (post_kernel-1)/2, -> out_channels)
 *   -> final_act (0 none, 1 clamp [-1, 1], 2 tanh).
 * The raw signal of an odd-stride ConvT stack is a few samples longer than
 * frames * hop (hop = product of the rates); y keeps the first frames * hop
 * samples of each row.
 * With tile_frames > 0 the latent is decoded in time tiles: tiles of
 * tile_frames frames start every tile_frames - overlap_frames frames, the
 * last one cut at `frames`; each tile is decoded as an independent signal
 * and trimmed to its own frames * hop samples; where tiles overlap, the
 * samples are averaged over the tiles covering them ([M3] windowed forward).
 * Tiles of equal length are batched into one decode.
 * Streams and threads: the AMP blocks of a stage run side by side on
 * library-owned streams (one set per device, forked from and joined back to
 * `stream` with events).  Calls from several host threads are safe: their
 * fork/join sequences are enqueued one at a time under a per-device lock,
 * and their blocks then share those streams.  While a decode is being
 * captured into a CUDA graph, no other thread may decode on that device
 * (its blocks would join the capture through the shared streams).
 * ---------------------------------------------------------------------- */
typedef struct {
  int in_channels;
  int pre_channels;
  int pre_kernel;
  int n_up;
  int up_rate[BV_MAX_UP];
  int up_kernel[BV_MAX_UP];
  int up_channels[BV_MAX_UP];
  int n_blocks;
  int block_kernel[BV_MAX_BLOCKS];
  int n_dilations;
  int dilation[BV_MAX_DIL];
  int post_kernel;
  int out_channels;
  int final_act;
  int tile_frames;     /* 0: decode the whole latent at once */
  int overlap_frames;  /* < tile_frames */
  int latent_channels; /* 0: z is the decoder's input [B, in_channels, frames].
                        * > 0: z holds normalised latents [latent_channels, B,
                        * frames] that first go through the latent front end
                        * (bv_latent_front_end) into in_channels */
  int tf32_only;       /* 0: the AMP-block convs and the transposed convs
                        * whose input channel count is a multiple of 8 from
                        * 48 up take their tensor-core operands as two fp16
                        * parts (x = hi + lo, W likewise,
                        * three products accumulated in fp32: 22 significant
                        * bits per operand as in the tf32 split, rounded
                        * instead of truncated, at twice the tf32 MMA rate);
                        * their activations must stay below 65504 in
                        * magnitude, else bv_sync_status reports BV_ERR_RANGE.
                        * 1: every tensor-core conv splits into tf32 parts
                        * (3xTF32, the full f32 range).  Prepared weights
                        * follow the config they were prepared with. */
} bv_decoder_config;

typedef struct {
  const float *pre_w, *pre_b;                 /* [pre_ch, in_ch, pre_k], [pre_ch] */
  const float *up_w[BV_MAX_UP], *up_b[BV_MAX_UP]; /* [Cin, Cout, k], [Cout] */
  bv_amp_params amp[BV_MAX_UP][BV_MAX_BLOCKS];
  const float *post_log_alpha, *post_log_beta; /* [C_last] */
  const float *post_w, *post_b;               /* [out_ch, C_last, post_k], [out_ch] */
  const float *up_filter, *down_filter;       /* [12] each, used by act_post */
  /* latent front end (used when latent_channels > 0): */
  const float *latents_mean, *latents_std;    /* [latent_channels] */
  const float *dec_in_w, *dec_in_b;           /* [in_ch, latent_ch, 1], [in_ch] or NULL */
  /* NULL, or a buffer bv_decoder_prepare wrote for this config and these
   * weight pointers: decodes then read the tensor-core weights from it
   * instead of splitting them into the workspace on every call */
  const void *prepared;
} bv_decoder_weights;

/* Prepared weights: the hi / lo split of every tensor-core conv's weights
 * (tap-major where the conv runs time-major; fp16 parts for the AMP convs the
 * config's tf32_only leaves on the fp16 split, else tf32) and the packed phase
 * weights of every tensor-core transposed conv, written once into a caller
 * buffer (device, 256-byte aligned, bv_decoder_prepared_size bytes) and read
 * by every later decode whose weights point at it (w->prepared).  The buffer
 * derives from the weight values at the time of the call: re-prepare after
 * changing them.  A decode with prepared weights needs only
 * bv_decode_workspace_size_prepared bytes of workspace.  Errors:
 * BV_ERR_ARG, BV_ERR_SHAPE, BV_ERR_WORKSPACE, BV_ERR_CUDA. */
size_t bv_decoder_prepared_size(const bv_decoder_config *cfg);
bv_status bv_decoder_prepare(const bv_decoder_config *cfg,
                             const bv_decoder_weights *w, void *prepared,
                             size_t bytes, void *stream);
size_t bv_decode_workspace_size_prepared(const bv_decoder_config *cfg, int B,
                                         int frames);

/* The latent front end of [H3] `AudioVae::decode`: normalised latents z
 * [C, S, T] (channel ci of side s at (ci S + s) T + t; the page's stereo
 * layout is S = 2) are de-normalised per channel and projected by
 * `dec_in_proj` ([H3] `AudioVae::from_cmf`: a Conv1d loaded with padding 0
 * whose output keeps the length, hence one tap):
 *   lat[s, ci, t] = z[ci, s, t] std[ci] + mean[ci],
 *   out[s, o, t]  = bias[o] + sum_ci w[o, ci] lat[s, ci, t].
 * z, mean, std, w [Cout, C, 1], bias [Cout] or NULL, out [S, Cout, T]: device.
 * out must not overlap z.  Errors: BV_ERR_ARG, BV_ERR_SHAPE (sizes < 1). */
bv_status bv_latent_front_end(const float *z, int C, int S, int T,
                              const float *mean, const float *std,
                              const float *w, const float *bias, int Cout,
                              float *out, void *stream);

/* Number of floats of the flat parameter vector of `cfg`, in module order:
 *  conv_pre w, b; per stage: ups w, b, then per block, per dilation:
 *  act1 log_alpha, log_beta, conv1 w, b, act2 log_alpha, log_beta, conv2 w, b;
 *  act_post log_alpha, log_beta; conv_post w, b.   -1 if cfg is invalid. */
int64_t bv_decoder_param_count(const bv_decoder_config *cfg);

/* Fills `out` with pointers into a flat DEVICE parameter vector laid out as
 * above; up_filter/down_filter ([12] device) go into every block and into
 * act_post.  Host-only pointer arithmetic. */
bv_status bv_decoder_weights_from_flat(const bv_decoder_config *cfg,
                                       const float *flat,
                                       const float *up_filter,
                                       const float *down_filter,
                                       bv_decoder_weights *out);

/* Samples per row of y: frames * product(up_rate). */
int64_t bv_decoder_output_length(const bv_decoder_config *cfg, int frames);

/* Workspace bytes bv_decode needs for B rows of `frames` latent frames
 * (0 if the request is invalid; see bv_last_error). */
size_t bv_decode_workspace_size(const bv_decoder_config *cfg, int B, int frames);

/* z [B, in_channels, frames] (or [latent_channels, B, frames] with the
 * latent front end) -> y [B, out_channels, frames * hop], device.
 * Errors: BV_ERR_ARG, BV_ERR_SHAPE, BV_ERR_WORKSPACE, BV_ERR_CUDA. */
bv_status bv_decode(const bv_decoder_config *cfg, const bv_decoder_weights *w,
                    const float *z, int B, int frames, float *y,
                    void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * The MiniMax-Music-3 DAV decoder ([H3] page, items `Snake`, `DavUnit`,
 * `DavStage`, `Music3Dav`):
 *   dec_in (one-tap Conv1d, latent_channels -> in_channels)
 *   -> conv_pre (pad (pre_kernel - 1)/2, -> pre_channels)
 *   -> for each stage i: Snake -> ConvT (rate up_rate[i], kernel
 *      up_kernel[i], pad (k - s)/2, exactly s samples per input sample,
 *      -> up_channels[i]) -> for each dilation d: x += c2(Snake(c1(Snake(x))))
 *      with c1 a unit_kernel-tap conv at dilation d (pad d (unit_kernel-1)/2)
 *      and c2 a one-tap conv
 *   -> Snake -> conv_post (pad (post_kernel - 1)/2) -> final_act.
 * Snake is the plain form with alpha used as stored:
 *   v = x + sin^2(alpha_c x) / (alpha_c + 1e-9).
 * The page's 128-channel latent is a stereo pair of 64: z [B = 2, 64, frames]
 * in this interface (its layout is already [2, 64, frames]); the result is
 * y [B, out_channels, frames * hop], hop = product of the rates (512 for
 * strides 8, 8, 4, 2).  Weights are device pointers in PyTorch layouts.
 * ---------------------------------------------------------------------- */
typedef struct {
  int latent_channels, in_channels, pre_channels, pre_kernel;
  int n_up;
  int up_rate[BV_MAX_UP], up_kernel[BV_MAX_UP], up_channels[BV_MAX_UP];
  int n_dilations;
  int dilation[BV_MAX_DIL];
  int unit_kernel, post_kernel, out_channels;
  int final_act; /* 0 none, 1 clamp [-1, 1], 2 tanh (the page's) */
} bv_dav_config;

typedef struct {
  const float *dec_in_w, *dec_in_b;      /* [in, latent, 1], [in] */
  const float *pre_w, *pre_b;            /* [pre, in, pre_k], [pre] */
  const float *stage_alpha[BV_MAX_UP];   /* [Cin_i] */
  const float *up_w[BV_MAX_UP], *up_b[BV_MAX_UP]; /* [Cin_i, Cout_i, k_i], [Cout_i] */
  const float *a1[BV_MAX_UP][BV_MAX_DIL], *c1_w[BV_MAX_UP][BV_MAX_DIL],
      *c1_b[BV_MAX_UP][BV_MAX_DIL];     /* [C], [C, C, unit_k], [C] */
  const float *a2[BV_MAX_UP][BV_MAX_DIL], *c2_w[BV_MAX_UP][BV_MAX_DIL],
      *c2_b[BV_MAX_UP][BV_MAX_DIL];     /* [C], [C, C, 1], [C] */
  const float *post_alpha, *post_w, *post_b; /* [C], [out, C, post_k], [out] */
} bv_dav_weights;

/* Floats of the flat parameter vector in module order: dec_in w, b; conv_pre
 * w, b; per stage: act alpha, up w, b, then per dilation a1 alpha, c1 w, b,
 * a2 alpha, c2 w, b; act_post alpha; conv_post w, b.  -1 if cfg is invalid
 * (including a stage whose kernel does not give exactly `rate` samples per
 * input sample). */
int64_t bv_dav_param_count(const bv_dav_config *cfg);
/* Pointers into a flat DEVICE parameter vector laid out as above. */
bv_status bv_dav_weights_from_flat(const bv_dav_config *cfg, const float *flat,
                                   bv_dav_weights *out);
int64_t bv_dav_output_length(const bv_dav_config *cfg, int frames);
size_t bv_dav_workspace_size(const bv_dav_config *cfg, int B, int frames);
/* z [B, latent_channels, frames] -> y [B, out_channels, frames * hop], all
 * device; z, y and the workspace disjoint.  Errors: BV_ERR_ARG,
 * BV_ERR_SHAPE, BV_ERR_WORKSPACE, BV_ERR_CUDA. */
bv_status bv_dav_decode(const bv_dav_config *cfg, const bv_dav_weights *w,
                        const float *z, int B, int frames, float *y,
                        void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------------
 * The LTX-2.5 bandwidth-extension tail ([LTX] `AudioStack::decode_from_mel`
 * after the first generator, `MelStft::forward`, `hann_sinc_upsample`).
 *
 * bv_mel_stft: the causal log-mel the extender reads.  x [C, T] is
 * left-padded with n_fft - hop zeros; frame f starts at f hop;
 *   frames = (T + n_fft - hop - n_fft) / hop + 1   (bv_mel_frames);
 *   re[r] = sum_j v[j] basis[r, j], im[r] = sum_j v[j] basis[n_freqs + r, j],
 *   out[c n_mels + m, f] = ln(max(sum_r mel_basis[m, r] |re + i im|, 1e-5)),
 * the (channel, mel) fold of [LTX] `Vocoder::forward`.  basis [2 n_freqs,
 * n_fft] (the checkpoint's DFT x window rows), mel_basis [n_mels, n_freqs],
 * out [C n_mels, frames]; device.
 *
 * bv_sinc_upsample: x [C, T] -> y [C, ratio T], the Hann-windowed sinc
 * interpolator (rolloff 0.99, 6 zero crossings, width = 7 input samples per
 * side, k = 2 width ratio + 1 float taps), the input replicate-padded by
 * width samples and scaled by ratio, a transposed FIR trimmed to
 * [2 width ratio, ...).
 *
 * bv_bwe_tail: low [C, T] at the input rate -> y [C, ratio T]:
 *   padded = low zero-padded to whole hops;
 *   y = clamp(extender(mel_stft(padded)) + sinc_upsample(padded), -1, 1)
 * over the first ratio T samples.  The extender is a decoder (cfg, w) run on
 * one row of C n_mels channels with C outputs (cfg: in_channels = C n_mels,
 * out_channels = C, final_act 0 as its output is a residual, untiled, no
 * latent front end, hop = ratio x mel hop).  Errors: BV_ERR_ARG,
 * BV_ERR_SHAPE, BV_ERR_WORKSPACE, BV_ERR_CUDA.
 * ---------------------------------------------------------------------- */
int64_t bv_mel_frames(int T, int n_fft, int hop);
bv_status bv_mel_stft(const float *x, int C, int T, const float *basis,
                      int n_freqs, int n_fft, int hop, const float *mel_basis,
                      int n_mels, float *out, void *stream);
bv_status bv_sinc_upsample(const float *x, int C, int T, int ratio, float *y,
                           void *stream);
size_t bv_bwe_tail_workspace_size(const bv_decoder_config *cfg, int C, int T,
                                  int n_fft, int hop, int n_mels, int ratio);
bv_status bv_bwe_tail(const bv_decoder_config *cfg, const bv_decoder_weights *w,
                      const float *low, int C, int T, const float *stft_basis,
                      int n_fft, int hop, const float *mel_basis, int n_mels,
                      int ratio, float *y, void *workspace, size_t ws_bytes,
                      void *stream);

/* ------------------------------------------------------------------------
 * The decode split into units, for sharding one decode over several GPUs
 * (each decodes a range of units, the outputs are gathered, one GPU
 * stitches).  Unit u = k * B + b is tile k of side b, in the tiling bv_decode
 * uses (an untiled decode is one tile of all `frames` frames).  A unit's row
 * holds out_channels x bv_decoder_unit_length samples: its tile's decoded
 * waveform, trimmed to the tile's frames * hop (a shorter last tile fills
 * only the front of its row; the rest of that row is unspecified).
 * Decoding every unit and stitching gives bv_decode's result bit for bit
 * (the units are decoded by the same kernels, rows independently).
 * ---------------------------------------------------------------------- */
/* Tiles of the tiling of `frames` (1 when untiled); -1 if invalid. */
int bv_decoder_tile_count(const bv_decoder_config *cfg, int frames);
/* Samples per unit row and output channel: tile_frames * hop (frames * hop
 * when untiled); -1 if invalid. */
int64_t bv_decoder_unit_length(const bv_decoder_config *cfg, int frames);
size_t bv_decode_units_workspace_size(const bv_decoder_config *cfg, int B,
                                      int frames, int64_t unit_begin,
                                      int64_t unit_end);
/* Decodes units [unit_begin, unit_end) of z [B, in_channels, frames] into
 * y_units [unit_end - unit_begin, out_channels, unit length] (unit u at row
 * u - unit_begin).  Errors as bv_decode; BV_ERR_SHAPE for a unit range
 * outside [0, tiles * B) or empty. */
bv_status bv_decode_units(const bv_decoder_config *cfg,
                          const bv_decoder_weights *w, const float *z, int B,
                          int frames, int64_t unit_begin, int64_t unit_end,
                          float *y_units, void *workspace, size_t ws_bytes,
                          void *stream);
/* y [B, out_channels, frames * hop] from all tiles * B unit rows in unit
 * order: each sample the mean of the tiles covering it ([M3] windowed
 * forward).  y_units and y must not overlap. */
bv_status bv_stitch_units(const bv_decoder_config *cfg, int B, int frames,
                          const float *y_units, float *y, void *stream);

/* bv_decode from HOST buffers: copies z_host (pinned for an asynchronous
 * copy) into the workspace, decodes, and copies the waveform back into
 * y_host, all on `stream`; the caller synchronises before reading y_host.
 * Workspace: bv_decode_host_workspace_size. */
size_t bv_decode_host_workspace_size(const bv_decoder_config *cfg, int B, int frames);
bv_status bv_decode_host(const bv_decoder_config *cfg,
                         const bv_decoder_weights *w, const float *z_host,
                         int B, int frames, float *y_host, void *workspace,
                         size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BV_H_ */
