// The MiniMax-Music-3 DAV decoder (docs.rs cortiq-engine 0.5.74 audiovae.rs,
// items `Snake`, `DavUnit`, `DavStage`, `Music3Dav`) on the library's conv
// kernels:
//   dec_in (one tap) -> conv_pre -> per stage: Snake -> ConvT (x stride) ->
//   residual units x += c2(Snake(c1(Snake(x)))) (c1 dilated, c2 one tap)
//   -> Snake -> conv_post -> final op,
// with the plain Snake v = x + sin^2(alpha x) / (alpha + 1e-9), alpha used as
// stored.  The Snake is pointwise, so where the next conv runs time-major on
// the tensor cores one pass applies it and writes that conv's tf32 hi / lo
// operand planes ([B, T, C]); elsewhere it writes [B, C, T].  The units'
// residual add is the second conv's epilogue, in place.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "sin2.cuh"

namespace bv {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

__device__ __forceinline__ float snake(float x, float a, float inv) {
  return fmaf(sin_squared(a * x), inv, x);
}

// y[r, t] = Snake(x[r, t]; alpha[r mod C]) over rows r of length T.
__global__ void __launch_bounds__(256) snake_kernel(const float *__restrict__ x,
                                                    float *__restrict__ y, int C, int T,
                                                    const float *__restrict__ alpha) {
  const int r = blockIdx.y;
  const float a = __ldg(alpha + r % C), inv = 1.0f / (a + 1e-9f);
  const float *xr = x + (size_t)r * T;
  float *yr = y + (size_t)r * T;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x)
    yr[t] = snake(__ldg(xr + t), a, inv);
}

// hi[b, t, c] = tf32(Snake(x[b, c, t])), lo = Snake(..) - hi: 32 x 32 tiles
// through shared memory, reads along t and writes along c coalesced.
__global__ void __launch_bounds__(256) snake_split_kernel(const float *__restrict__ x,
                                                          float *__restrict__ hi,
                                                          float *__restrict__ lo, int C, int T,
                                                          const float *__restrict__ alpha) {
  __shared__ float tile[32][33];
  const int t0 = blockIdx.x * 32, c0 = blockIdx.y * 32, b = blockIdx.z;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const float *xb = x + (size_t)b * C * T;
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int t = t0 + tx, c = c0 + r;
    float v = 0.0f;
    if (t < T && c < C) {
      const float a = __ldg(alpha + c);
      v = snake(__ldg(xb + (size_t)c * T + t), a, 1.0f / (a + 1e-9f));
    }
    tile[r][tx] = v;
  }
  __syncthreads();
  const size_t ob = (size_t)b * T * C;
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int t = t0 + r;
    if (t < T && c0 + tx < C) {
      const float v = tile[tx][r];
      const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
      const size_t idx = ob + (size_t)t * C + c0 + tx;
      hi[idx] = h;
      lo[idx] = v - h;
    }
  }
}

bv_status launch_snake(const float *x, float *y, int B, int C, int T, const float *alpha,
                       cudaStream_t st) {
  if (B <= 0 || C <= 0 || T <= 0) return BV_OK;
  const int rows = B * C;
  if (rows > 65535) return fail(BV_ERR_SHAPE, "snake: %d rows", rows);
  const int bx = std::min((T + 255) / 256, 64);
  {
    LaunchTimer tm(st, "snake", 0.0, 8.0 * (double)rows * T);
    snake_kernel<<<dim3(bx, rows), 256, 0, st>>>(x, y, C, T, alpha);
  }
  count_launch();
  return check_launch("snake_kernel");
}

bv_status launch_snake_split(const float *x, float *hi, float *lo, int B, int C, int T,
                             const float *alpha, cudaStream_t st) {
  if (B <= 0 || C <= 0 || T <= 0) return BV_OK;
  dim3 grid((T + 31) / 32, (C + 31) / 32, B);
  if (grid.y > 65535 || grid.z > 65535) return fail(BV_ERR_SHAPE, "snake_split: grid");
  {
    LaunchTimer tm(st, "snake_split", 0.0, 12.0 * (double)B * C * T);
    snake_split_kernel<<<grid, 256, 0, st>>>(x, hi, lo, C, T, alpha);
  }
  count_launch();
  return check_launch("snake_split_kernel");
}

bv_status check_dav_config(const bv_dav_config *c) {
  if (!c) return fail(BV_ERR_ARG, "dav: null config");
  if (c->latent_channels < 1 || c->in_channels < 1 || c->pre_channels < 1 || c->out_channels < 1)
    return fail(BV_ERR_SHAPE, "dav: channel counts must be >= 1");
  if (c->pre_kernel < 1 || c->pre_kernel % 2 == 0 || c->pre_kernel > 31 || c->post_kernel < 1 ||
      c->post_kernel % 2 == 0 || c->post_kernel > 31 || c->unit_kernel < 1 ||
      c->unit_kernel % 2 == 0 || c->unit_kernel > 31)
    return fail(BV_ERR_SHAPE, "dav: pre/unit/post kernels must be odd and <= 31");
  if (c->n_up < 0 || c->n_up > BV_MAX_UP) return fail(BV_ERR_SHAPE, "dav: n_up %d", c->n_up);
  for (int i = 0; i < c->n_up; ++i) {
    const int s = c->up_rate[i], k = c->up_kernel[i];
    // every stage must give exactly `s` samples per input sample, as the
    // page's `n = n * stride` assumes: k - 2 (k - s)/2 == s
    if (s < 1 || s > 16 || k < s || k > 64 || c->up_channels[i] < 1 || k - 2 * ((k - s) / 2) != s)
      return fail(BV_ERR_SHAPE, "dav: stage %d rate %d kernel %d channels %d", i, s, k,
                  c->up_channels[i]);
  }
  if (c->n_dilations < 0 || c->n_dilations > BV_MAX_DIL)
    return fail(BV_ERR_SHAPE, "dav: n_dilations %d", c->n_dilations);
  for (int u = 0; u < c->n_dilations; ++u)
    if (c->dilation[u] < 1) return fail(BV_ERR_SHAPE, "dav: dilation %d", c->dilation[u]);
  if (c->final_act < 0 || c->final_act > 2) return fail(BV_ERR_ARG, "dav: final_act %d", c->final_act);
  return BV_OK;
}

long long dav_hop(const bv_dav_config *c) {
  long long h = 1;
  for (int i = 0; i < c->n_up; ++i) h *= c->up_rate[i];
  return h;
}

// Largest B C T over the decoder's stored tensors (z excluded).
long long dav_max_elems(const bv_dav_config *c, long long B, long long F) {
  long long m = B * std::max(c->in_channels, c->pre_channels) * F, n = F;
  for (int i = 0; i < c->n_up; ++i) {
    n *= c->up_rate[i];
    m = std::max(m, B * c->up_channels[i] * n);
  }
  return m;
}

// The unit convs that run time-major: c1 (unit_kernel taps) and c2 (one tap)
// of each stage, by channel count and dilation.
bool dav_c1_tm(const bv_dav_config *c, int C, int d) {
  return conv1d_tm_supported(C, C, c->unit_kernel, d);
}
bool dav_c2_tm(int C) { return conv1d_tm_supported(C, C, 1, 1); }

size_t split_bytes(int Cin, int Cout, int K) {
  return align_up(2 * (size_t)tm_cin_pad(Cin) * Cout * K * sizeof(float));
}

size_t dav_split_ws(const bv_dav_config *c) {
  size_t s = 0;
  for (int i = 0; i < c->n_up; ++i) {
    const int C = c->up_channels[i];
    for (int u = 0; u < c->n_dilations; ++u) {
      if (dav_c1_tm(c, C, c->dilation[u])) s += split_bytes(C, C, c->unit_kernel);
      if (dav_c2_tm(C)) s += split_bytes(C, C, 1);
    }
  }
  return s;
}

size_t dav_convt_ws(const bv_dav_config *c) {
  size_t m = 0;
  int C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const int Co = c->up_channels[i], k = c->up_kernel[i], s = c->up_rate[i];
    if (conv_transpose1d_tm_supported(C, Co, k, s))
      m = std::max(m, conv_transpose1d_tm_workspace(C, Co, k, s));
    else if (conv_transpose1d_tc_supported(C, Co, k, s))
      m = std::max(m, conv_transpose1d_tc_workspace(C, Co, k, s));
    C = Co;
  }
  return align_up(m);
}

// Buffers of max_elems floats: X (running signal), S (ConvT output), H (c1
// output), A (a Snake output in [B, C, T]), P_hi, P_lo (time-major planes).
constexpr int kDavPlanes = 6;

size_t dav_ws(const bv_dav_config *c, int B, int F) {
  return dav_split_ws(c) +
         kDavPlanes * align_up((size_t)dav_max_elems(c, B, F) * sizeof(float)) + dav_convt_ws(c);
}

bv_status check_dav_weights(const bv_dav_config *c, const bv_dav_weights *w) {
  if (!w) return fail(BV_ERR_ARG, "dav: null weights");
  if (!w->dec_in_w || !w->pre_w || !w->post_alpha || !w->post_w)
    return fail(BV_ERR_ARG, "dav: null dec_in / conv_pre / act_post / conv_post weight");
  for (int i = 0; i < c->n_up; ++i) {
    if (!w->stage_alpha[i] || !w->up_w[i]) return fail(BV_ERR_ARG, "dav: null stage %d weight", i);
    for (int u = 0; u < c->n_dilations; ++u)
      if (!w->a1[i][u] || !w->c1_w[i][u] || !w->a2[i][u] || !w->c2_w[i][u])
        return fail(BV_ERR_ARG, "dav: null weight in stage %d unit %d", i, u);
  }
  return BV_OK;
}

bv_status dav_decode_impl(const bv_dav_config *c, const bv_dav_weights *w, const float *z,
                          int B, int F, float *y, char *ws, cudaStream_t st) {
  // tap-major tf32 hi / lo weights of the time-major unit convs
  const float *c1s[BV_MAX_UP][BV_MAX_DIL] = {}, *c2s[BV_MAX_UP][BV_MAX_DIL] = {};
  {
    SplitTable tab;
    tab.n = 0;
    size_t off = 0;
    auto add = [&](const float *src, int C, int K, const float **slot) -> bv_status {
      float *dst = reinterpret_cast<float *>(ws + off);
      off += split_bytes(C, C, K);
      *slot = dst;
      tab.src[tab.n] = src;
      tab.dst[tab.n] = dst;
      tab.count[tab.n] = (long long)C * C * K;
      tab.cin[tab.n] = C;
      tab.k[tab.n] = K;
      tab.f16[tab.n] = 0;  // the DAV convs read tf32 planes
      if (++tab.n == kMaxSplit) {
        BV_TRY(launch_split_weights(tab, st));
        tab.n = 0;
      }
      return BV_OK;
    };
    for (int i = 0; i < c->n_up; ++i) {
      const int C = c->up_channels[i];
      for (int u = 0; u < c->n_dilations; ++u) {
        if (dav_c1_tm(c, C, c->dilation[u])) BV_TRY(add(w->c1_w[i][u], C, c->unit_kernel, &c1s[i][u]));
        if (dav_c2_tm(C)) BV_TRY(add(w->c2_w[i][u], C, 1, &c2s[i][u]));
      }
    }
    BV_TRY(launch_split_weights(tab, st));
    ws += dav_split_ws(c);
  }
  const size_t sz = align_up((size_t)dav_max_elems(c, B, F) * sizeof(float));
  auto plane = [&](int k) { return reinterpret_cast<float *>(ws + (size_t)k * sz); };
  float *X = plane(0), *S = plane(1), *H = plane(2), *A = plane(3), *Ph = plane(4), *Pl = plane(5);
  float *WP = plane(kDavPlanes);
  const Epi plain{nullptr, 1.0f, 0, 0};
  // dec_in (one tap) into A, conv_pre into X
  BV_TRY(launch_conv1d(z, B, c->latent_channels, F, w->dec_in_w, w->dec_in_b, c->in_channels, 1,
                       1, 0, plain, A, F, F, st));
  BV_TRY(launch_conv1d(A, B, c->in_channels, F, w->pre_w, w->pre_b, c->pre_channels,
                       c->pre_kernel, 1, (c->pre_kernel - 1) / 2, plain, X, F, F, st));
  int C = c->pre_channels, n = F;
  for (int i = 0; i < c->n_up; ++i) {
    const int s = c->up_rate[i], k = c->up_kernel[i], Co = c->up_channels[i];
    const int pad = (k - s) / 2;
    // Snake -> ConvT into S
    if (conv_transpose1d_tm_supported(C, Co, k, s)) {
      BV_TRY(launch_snake_split(X, Ph, Pl, B, C, n, w->stage_alpha[i], st));
      BV_TRY(launch_conv_transpose1d_tm(Ph, Pl, B, C, n, w->up_w[i], w->up_b[i], Co, k, s, pad, S,
                                        WP, st));
    } else {
      BV_TRY(launch_snake(X, A, B, C, n, w->stage_alpha[i], st));
      if (conv_transpose1d_tc_supported(C, Co, k, s))
        BV_TRY(launch_conv_transpose1d_tc(A, B, C, n, w->up_w[i], w->up_b[i], Co, k, s, pad, S,
                                          WP, st));
      else
        BV_TRY(launch_conv_transpose1d(A, B, C, n, w->up_w[i], w->up_b[i], Co, k, s, pad, S, st));
    }
    std::swap(X, S);
    C = Co;
    n *= s;
    for (int u = 0; u < c->n_dilations; ++u) {
      const int d = c->dilation[u], K = c->unit_kernel;
      const int pu = d * (K - 1) / 2;
      // h = c1(Snake(x; a1)) into H
      if (c1s[i][u]) {
        BV_TRY(launch_snake_split(X, Ph, Pl, B, C, n, w->a1[i][u], st));
        BV_TRY(launch_conv1d_tm(Ph, Pl, B, C, n, c1s[i][u], w->c1_b[i][u], C, K, d, pu, plain, H, n,
                                n, st));
      } else {
        BV_TRY(launch_snake(X, A, B, C, n, w->a1[i][u], st));
        BV_TRY(launch_conv1d(A, B, C, n, w->c1_w[i][u], w->c1_b[i][u], C, K, d, pu, plain, H, n, n,
                             st));
      }
      // x += c2(Snake(h; a2)), the residual add in the epilogue, in place
      const Epi res{X, 1.0f, 0, 0};
      if (c2s[i][u]) {
        BV_TRY(launch_snake_split(H, Ph, Pl, B, C, n, w->a2[i][u], st));
        BV_TRY(launch_conv1d_tm(Ph, Pl, B, C, n, c2s[i][u], w->c2_b[i][u], C, 1, 1, 0, res, X, n,
                                n, st));
      } else {
        BV_TRY(launch_snake(H, A, B, C, n, w->a2[i][u], st));
        BV_TRY(launch_conv1d(A, B, C, n, w->c2_w[i][u], w->c2_b[i][u], C, 1, 1, 0, res, X, n, n, st));
      }
    }
  }
  BV_TRY(launch_snake(X, A, B, C, n, w->post_alpha, st));
  const Epi fin{nullptr, 1.0f, 0, c->final_act};
  return launch_conv1d(A, B, C, n, w->post_w, w->post_b, c->out_channels, c->post_kernel, 1,
                       (c->post_kernel - 1) / 2, fin, y, n, n, st);
}

}  // namespace
}  // namespace bv

using namespace bv;

extern "C" {

int64_t bv_dav_param_count(const bv_dav_config *c) {
  if (check_dav_config(c) != BV_OK) return -1;
  int64_t n = (int64_t)c->in_channels * c->latent_channels + c->in_channels;
  n += (int64_t)c->pre_channels * c->in_channels * c->pre_kernel + c->pre_channels;
  int64_t C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const int64_t Co = c->up_channels[i];
    n += C + C * Co * c->up_kernel[i] + Co;
    n += (int64_t)c->n_dilations * (2 * Co + Co * Co * c->unit_kernel + Co + Co * Co + Co);
    C = Co;
  }
  return n + C + (int64_t)c->out_channels * C * c->post_kernel + c->out_channels;
}

bv_status bv_dav_weights_from_flat(const bv_dav_config *c, const float *flat,
                                   bv_dav_weights *out) {
  clear_error();
  BV_TRY(check_dav_config(c));
  if (!flat || !out) return fail(BV_ERR_ARG, "bv_dav_weights_from_flat: null pointer");
  std::memset(out, 0, sizeof(*out));
  const float *p = flat;
  auto take = [&](size_t n) {
    const float *q = p;
    p += n;
    return q;
  };
  out->dec_in_w = take((size_t)c->in_channels * c->latent_channels);
  out->dec_in_b = take(c->in_channels);
  out->pre_w = take((size_t)c->pre_channels * c->in_channels * c->pre_kernel);
  out->pre_b = take(c->pre_channels);
  size_t C = c->pre_channels;
  for (int i = 0; i < c->n_up; ++i) {
    const size_t Co = c->up_channels[i];
    out->stage_alpha[i] = take(C);
    out->up_w[i] = take(C * Co * c->up_kernel[i]);
    out->up_b[i] = take(Co);
    C = Co;
    for (int u = 0; u < c->n_dilations; ++u) {
      out->a1[i][u] = take(C);
      out->c1_w[i][u] = take(C * C * c->unit_kernel);
      out->c1_b[i][u] = take(C);
      out->a2[i][u] = take(C);
      out->c2_w[i][u] = take(C * C);
      out->c2_b[i][u] = take(C);
    }
  }
  out->post_alpha = take(C);
  out->post_w = take((size_t)c->out_channels * C * c->post_kernel);
  out->post_b = take(c->out_channels);
  return BV_OK;
}

int64_t bv_dav_output_length(const bv_dav_config *c, int frames) {
  if (check_dav_config(c) != BV_OK || frames < 1) return -1;
  return (int64_t)frames * dav_hop(c);
}

size_t bv_dav_workspace_size(const bv_dav_config *c, int B, int frames) {
  clear_error();
  if (check_dav_config(c) != BV_OK) return 0;
  if (B < 1 || frames < 1) {
    fail(BV_ERR_SHAPE, "bv_dav_workspace_size: B=%d frames=%d", B, frames);
    return 0;
  }
  return dav_ws(c, B, frames);
}

bv_status bv_dav_decode(const bv_dav_config *c, const bv_dav_weights *w, const float *z, int B,
                        int frames, float *y, void *workspace, size_t ws_bytes, void *stream) {
  clear_error();
  BV_TRY(check_dav_config(c));
  if (!z || !y) return fail(BV_ERR_ARG, "bv_dav_decode: null z or y");
  if (B < 1 || frames < 1) return fail(BV_ERR_SHAPE, "bv_dav_decode: B=%d frames=%d", B, frames);
  const long long L = (long long)frames * dav_hop(c);
  if (L > 0x7fffffffLL || dav_max_elems(c, B, frames) > (1LL << 40))
    return fail(BV_ERR_SHAPE, "bv_dav_decode: request too large");
  BV_TRY(check_dav_weights(c, w));
  const size_t need = dav_ws(c, B, frames);
  if (!workspace || ws_bytes < need)
    return fail(BV_ERR_WORKSPACE, "bv_dav_decode: workspace %zu bytes, need %zu", ws_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
    return fail(BV_ERR_ARG, "bv_dav_decode: workspace not 256-byte aligned");
  const size_t nz = (size_t)B * c->latent_channels * frames, ny = (size_t)B * c->out_channels * L;
  const float *wsf = static_cast<const float *>(workspace);
  if (overlaps(z, nz, y, ny) || overlaps(z, nz, wsf, need / 4) || overlaps(y, ny, wsf, need / 4))
    return fail(BV_ERR_ARG, "bv_dav_decode: z, y and workspace must be disjoint");
  BV_TRY(require_device());
  return dav_decode_impl(c, w, z, B, frames, y, static_cast<char *>(workspace),
                         as_stream(stream));
}

}  // extern "C"
