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
  BV_ERR_UNSUPPORTED = 6  /* a valid request this build does not implement */
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
 * set when they give up; returns BV_OK or BV_ERR_TIMEOUT.  Synchronises
 * `stream`. */
bv_status bv_sync_status(void *stream);

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
 * two [B, T, C] operand planes and the convs' weights split into tf32 hi / lo
 * parts, besides the three [B, C, T] buffers.  Equals
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
} bv_decoder_config;

typedef struct {
  const float *pre_w, *pre_b;                 /* [pre_ch, in_ch, pre_k], [pre_ch] */
  const float *up_w[BV_MAX_UP], *up_b[BV_MAX_UP]; /* [Cin, Cout, k], [Cout] */
  bv_amp_params amp[BV_MAX_UP][BV_MAX_BLOCKS];
  const float *post_log_alpha, *post_log_beta; /* [C_last] */
  const float *post_w, *post_b;               /* [out_ch, C_last, post_k], [out_ch] */
  const float *up_filter, *down_filter;       /* [12] each, used by act_post */
} bv_decoder_weights;

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

/* z [B, in_channels, frames] -> y [B, out_channels, frames * hop], device.
 * Errors: BV_ERR_ARG, BV_ERR_SHAPE, BV_ERR_WORKSPACE, BV_ERR_CUDA. */
bv_status bv_decode(const bv_decoder_config *cfg, const bv_decoder_weights *w,
                    const float *z, int B, int frames, float *y,
                    void *workspace, size_t ws_bytes, void *stream);

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
