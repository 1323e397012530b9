// Dilated Conv1d as an implicit GEMM on the 5th-generation tensor cores
// (tcgen05, accumulator in TMEM), with FP32 accuracy from a 3xTF32 split.
//
//   y[b,o,t] = bias[o] + sum_i sum_j w[o,i,j] x[b,i,t + j d - pad]
// (docs.rs cortiq-engine audiovae.rs `Conv1d::apply`, whose note states the
// im2col identity used here; ltxaudio.rs `Conv1d::forward`).
//
// GEMM view: D[t, o] = sum_kk X[t, kk] W[o, kk] with kk = i K + j (the order of
// w's own [Cout][Cin][K] layout, so W is w read as a [Cout, Cin K] matrix) and
// X[t, kk] = x[b, i, t + j d - pad] (im2col, never materialised).  Time is the
// MMA's M side (128 per CTA) and output channels its N side (NT per CTA, a
// multiple of 16 sized to Cout, so narrow layers waste no tensor work).
// Each CTA walks kk in chunks of 32 (one 128-byte swizzle row of fp32):
//   - TMA brings the weight chunk W [NT x 32] into a ring of raw slots;
//   - four converter warps split it into W_hi = tf32(W) (low 13 mantissa bits
//     cleared) and W_lo = W - W_hi, and build X_hi / X_lo [128 t x 32 kk] from
//     input rows staged in shared memory with cp.async, all in the K-major
//     128-byte-swizzled layout the tensor core reads;
//   - one thread issues three tcgen05.mma.kind::tf32 per 8-wide k step,
//     X_lo W_hi + X_hi W_lo + X_hi W_hi, into an FP32 TMEM accumulator (the
//     3xTF32 scheme: the dropped X_lo W_lo term is 2^-22 relative);
//   - runs of RUN chunks accumulate in one of two TMEM accumulators starting
//     from zero, and the converter warps add each finished run into FP32
//     registers: the tensor core's accumulation truncates, so its error would
//     otherwise grow with Cin K;
//   - the epilogue (bias, residual, scale, accumulate, final op) has one
//     thread per time sample, so global reads and writes are coalesced.
// Two operand stages overlap conversion with the MMAs.  Every mbarrier wait
// is bounded (wait_limit polls, a kernel argument); a wait that runs out sets
// the device status word and marks the CTA aborted.  Aborting is orderly:
// each role stops issuing work at its first failed wait, every producer then
// waits (with a fixed bound) for the copies it issued, the MMA issuer waits
// for a final commit that covers all its MMAs, and only then is TMEM freed;
// the output tile is left unspecified.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace bv {
namespace {

constexpr int BM = 128;                  // time samples per CTA (UMMA M)
constexpr int MAX_NT = 128;              // output channels per CTA (UMMA N), at most
constexpr int BK = 32;                   // kk per chunk
constexpr int NSTAGE = 2;                // operand stages
constexpr int NRAW = 2;                  // TMA ring of raw weight chunks
constexpr int CB = 32;                   // input channels per staged x block
constexpr int MAX_HALO = 56;             // (K - 1) d the staged rows can hold
constexpr int XW = BM + MAX_HALO + 8;    // staged row width (floats)
constexpr int X_TILE = BM * BK * 4;      // 16 KB: one im2col operand tile
constexpr int W_TILE = MAX_NT * BK * 4;  // 16 KB: one weight operand tile (at most)
constexpr int THREADS = 256;
constexpr int CONV_WARP0 = 4;            // warps 4..7 convert, add runs, write out
constexpr int NCONV = 128;
constexpr long long DRAIN_LIMIT = 1ll << 22;  // polls for in-flight copies when unwinding
constexpr int TMEM_COLS = 256;           // two accumulators of up to 128 columns
constexpr int RUN = 4;                   // chunks accumulated in TMEM before an FP32 add
constexpr int MAX_K = 32;                // largest kernel size (offset table rows)

// shared memory layout (bytes from a 1024-aligned base): im2col operand
// stages, then a weight region of six 16 KB tiles, then the staged x blocks.
// The weight region holds W_hi[2], W_lo[2] and the raw TMA ring[2] when the
// kernel splits the weights itself, or W_hi[3], W_lo[3] (a three-slot TMA
// ring) when the split weights come from global memory.
constexpr int NWSLOT = 3;                                // pre-split weight ring
constexpr int OFF_XHI = 0;                               // per operand stage
constexpr int OFF_XLO = OFF_XHI + NSTAGE * X_TILE;
constexpr int OFF_W = OFF_XLO + NSTAGE * X_TILE;         // weight region
constexpr int OFF_X = OFF_W + 6 * W_TILE;                // x blocks [2][CB][XW]
static_assert(NSTAGE * 2 + NRAW == 6 && NWSLOT * 2 == 6, "weight region layout");
template <bool PRESPLIT>
struct WLayout {
  __host__ __device__ static constexpr int hi(int s) { return OFF_W + s * W_TILE; }
  __host__ __device__ static constexpr int lo(int s) { return OFF_W + (PRESPLIT ? NWSLOT : NSTAGE) * W_TILE + s * W_TILE; }
  __host__ __device__ static constexpr int raw(int r) { return OFF_W + 2 * NSTAGE * W_TILE + r * W_TILE; }
};
constexpr int X_BYTES = 2 * CB * XW * 4;
constexpr int OFF_BAR = OFF_X + X_BYTES;                 // mbarriers
constexpr int SMEM_USED = OFF_BAR + 16 * 8;
constexpr int SMEM_BYTES = SMEM_USED + 1024;             // room to align the base
static_assert(SMEM_BYTES + 4 * 1024 + 1024 <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ unsigned smem_u32(const void *p) {
  return (unsigned)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(unsigned bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of an mbarrier phase: cheaper than try_wait when the
// phase has already completed (measured on B200: ~160 against ~280 cycles in
// the MMA issuer's wait for a weight chunk that had landed long before).
__device__ __forceinline__ bool mbar_test(unsigned bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

struct Ctl {
  int abort;      // a bounded wait gave up somewhere in the CTA (or its pair)
  unsigned tmem;  // TMEM base address from tcgen05.alloc
};

// How a CTA reports a wait that ran out: its own Ctl, the shared::cluster
// address of its pair peer's abort flag (0 for a lone CTA), the device status
// word and the poll limit.
struct WaitCtx {
  volatile Ctl *ctl;
  unsigned peer_abort;
  int *status;
  long long limit;
};

__device__ __forceinline__ void raise_abort(const WaitCtx &w, int code) {
  w.ctl->abort = 1;
  if (w.peer_abort)
    asm volatile("st.shared::cluster.u32 [%0], %1;\n" ::"r"(w.peer_abort), "r"(1) : "memory");
  if (w.status) atomicExch(w.status, code);
}

// Bounded wait on an mbarrier phase: true once the phase has completed;
// false after w.limit polls (the CTA and its peer are then marked aborted and
// the failure recorded in the device status word) or once an abort raised
// elsewhere in the pair is seen.  A role stops issuing work at its first
// false.
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity, const WaitCtx &w,
                                          int code) {
  if (mbar_test(bar, parity)) return true;
  for (long long it = 0; it < w.limit; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255) == 255 && w.ctl->abort) return false;
  }
  raise_abort(w, code);
  return false;
}

// Wait with a fixed bound that does not return early on abort: used to let
// the copies and MMAs a role issued finish before the CTA frees TMEM or exits.
__device__ __forceinline__ void mbar_drain(unsigned bar, unsigned parity) {
  for (long long it = 0; it < DRAIN_LIMIT; ++it)
    if (mbar_try_wait(bar, parity)) return;
}

// Converter-side wait: lane 0 polls the barrier, the warp follows it, so the
// polling does not compete with the conversion for shared-memory bandwidth;
// the outcome is the same for every lane.
__device__ __forceinline__ bool warp_wait(unsigned bar, unsigned parity, const WaitCtx &w,
                                          int code) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, w, code) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void cp_async4_zfill(float *dst, const float *src, bool valid) {
  const unsigned d = smem_u32(dst);
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}
__device__ __forceinline__ void conv_bar_sync() {  // the four converter warps
  asm volatile("bar.sync 1, %0;\n" ::"n"(NCONV) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(unsigned addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: D f32, A and B tf32, both K-major, M = 128, N = nt.
__host__ __device__ constexpr uint32_t make_idesc(int nt) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(nt >> 3) << 17) |
         ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(unsigned tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         unsigned acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(unsigned bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
      : "memory");
}

// Byte offset of element (row r, column k < 32) in a K-major SW128 tile of
// 128-byte rows: 8-row groups of 1024 bytes, 16-byte chunk index XOR (r % 8).
__device__ __forceinline__ int sw128_off(int r, int k) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((((k >> 2) ^ (r & 7))) << 4) + ((k & 3) << 2);
}

__device__ __forceinline__ float tf32_hi(float v) {
  return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
}

// Where conv output t goes: sample stride * t + offset of a row of len
// samples; phases > 1 runs that many weight sets (blockIdx.z = b phases + r),
// phase r reading weight rows r Cout .. and writing offset + r.
struct OutMap {
  int stride, offset, len, phases;
};

template <int NT, bool PRESPLIT>
__global__ void __launch_bounds__(THREADS, 1)
conv1d_tc_kernel(const __grid_constant__ CUtensorMap tmap_w,
                 const __grid_constant__ CUtensorMap tmap_wlo, const float *__restrict__ x,
                 const float *__restrict__ bias, float *y, int Cin, int T, int Cout, int K,
                 int dil, int pad, int y_len, int y_pitch, Epi ep, OutMap om, int *status,
                 long long wait_limit) {
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= MAX_NT, "UMMA N for M = 128");
  constexpr int W_BYTES = NT * BK * 4;  // bytes of one weight chunk (TMA box)
  constexpr uint32_t IDESC = make_idesc(NT);
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  __shared__ Ctl ctl;
  __shared__ float bias_s[MAX_NT];  // this tile's biases (0 past Cout or without bias)
  __shared__ __align__(16) int xoff[MAX_K * BK];  // im2col offsets of chunk m of a block
  using WL = WLayout<PRESPLIT>;
  constexpr int NWRING = PRESPLIT ? NWSLOT : NRAW;  // weight TMA ring slots
  // barriers: weights landed (TMA) / weight slot free, per ring slot;
  // operands ready / operand stage free, per stage; run accumulated / run
  // accumulator read, per TMEM accumulator
  const unsigned bar_full_w = smem_u32(&bars[0]);
  const unsigned bar_raw_free = smem_u32(&bars[3]);
  const unsigned bar_ready = smem_u32(&bars[6]);
  const unsigned bar_empty = smem_u32(&bars[8]);
  const unsigned bar_run_full = smem_u32(&bars[10]);
  const unsigned bar_run_free = smem_u32(&bars[12]);
  const unsigned bar_done = smem_u32(&bars[14]);  // every MMA of the CTA has completed
  float *xs = reinterpret_cast<float *>(smem + OFF_X);
  const WaitCtx wc{&ctl, 0u, status, wait_limit};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * BM;
  const int o0 = blockIdx.y * NT;
  const int b = blockIdx.z / om.phases;
  const int phase = blockIdx.z - b * om.phases;
  const int w_row0 = phase * Cout + o0;  // this phase's weight rows in the tensor map
  const int KK = Cin * K;
  const int n_chunks = (KK + BK - 1) / BK;
  const int n_runs = (n_chunks + RUN - 1) / RUN;
  const int halo = (K - 1) * dil;
  const int xt0 = t0 - pad;  // time of staged column 0

  if (threadIdx.x == 0) {
    ctl.abort = 0;
    for (int s = 0; s < NWRING; ++s) {
      mbar_init(bar_full_w + 8 * s, 1);
      // a pre-split slot is freed by the MMA's commit, a raw slot by the converters
      mbar_init(bar_raw_free + 8 * s, PRESPLIT ? 1 : NCONV / 32);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_ready + 8 * s, NCONV / 32);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_run_full + 8 * s, 1);
      mbar_init(bar_run_free + 8 * s, NCONV / 32);
    }
    mbar_init(bar_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  // chunk m of an x block covers block-local kk = 32 m + e = i K + j
  for (int idx = threadIdx.x; idx < K * BK; idx += THREADS) {
    const int i = idx / K, j = idx - i * K;
    xoff[idx] = i * XW + j * dil;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&ctl.tmem)),
                 "n"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  for (int i = threadIdx.x; i < MAX_NT; i += THREADS)
    bias_s[i] = (bias && o0 + i < Cout) ? bias[o0 + i] : 0.0f;
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const unsigned tmem = ctl.tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % NWRING, u = c / NWRING;
        // A raw slot is free once the converters have split the chunk it
        // held; a pre-split slot once the MMAs that read it have finished.
        // On a failed wait no further load is issued.
        if (u > 0 && !mbar_wait(bar_raw_free + 8 * s, (u - 1) & 1, wc, 101)) break;
        const unsigned dst = smem_u32(smem + (PRESPLIT ? WL::hi(s) : WL::raw(s)));
        mbar_arrive_tx(bar_full_w + 8 * s, PRESPLIT ? 2 * W_BYTES : W_BYTES);
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
            "l"(reinterpret_cast<uint64_t>(&tmap_w)), "r"(c * BK), "r"(w_row0),
            "r"(bar_full_w + 8 * s)
            : "memory");
        if (PRESPLIT)
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_u32(smem + WL::lo(s))),
              "l"(reinterpret_cast<uint64_t>(&tmap_wlo)), "r"(c * BK), "r"(w_row0),
              "r"(bar_full_w + 8 * s)
              : "memory");
        issued = c + 1;
      }
      // drain: every slot holds at most one load not yet seen complete, the
      // last one issued into it; it must land before the CTA can exit
      for (int c = issued - NWRING; c < issued; ++c)
        if (c >= 0) mbar_drain(bar_full_w + 8 * (c % NWRING), (c / NWRING) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      for (int c = 0; c < n_chunks; ++c) {
        const int s = c % NSTAGE, u = c / NSTAGE;
        const int r = c / RUN, ra = r & 1;
        const bool first = (c % RUN) == 0;
        const bool last = (c % RUN) == RUN - 1 || c == n_chunks - 1;
        // the converters have read this accumulator's run r - 2
        if (first && r >= 2 && !mbar_wait(bar_run_free + 8 * ra, ((r >> 1) - 1) & 1, wc, 106))
          break;
        if (!mbar_wait(bar_ready + 8 * s, u & 1, wc, 102)) break;
        const int ws = PRESPLIT ? c % NWSLOT : s;  // weight slot of this chunk
        if (PRESPLIT && !mbar_wait(bar_full_w + 8 * ws, (c / NWSLOT) & 1, wc, 107)) break;
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        const unsigned acc = tmem + (unsigned)(ra * MAX_NT);
        const unsigned x_hi = smem_u32(smem + OFF_XHI + s * X_TILE);
        const unsigned x_lo = smem_u32(smem + OFF_XLO + s * X_TILE);
        const unsigned w_hi = smem_u32(smem + WL::hi(ws));
        const unsigned w_lo = smem_u32(smem + WL::lo(ws));
#pragma unroll
        for (int k = 0; k < BK / 8; ++k) {  // 8 tf32 = 32 bytes per MMA
          const unsigned off = 32 * k;
          mma_tf32(acc, sw128_desc(x_lo + off), sw128_desc(w_hi + off), IDESC,
                   (first && k == 0) ? 0u : 1u);
          mma_tf32(acc, sw128_desc(x_hi + off), sw128_desc(w_lo + off), IDESC, 1u);
          mma_tf32(acc, sw128_desc(x_hi + off), sw128_desc(w_hi + off), IDESC, 1u);
        }
        mma_commit(bar_empty + 8 * s);  // stage s may be refilled once these finish
        if (PRESPLIT) mma_commit(bar_raw_free + 8 * ws);  // and the weight slot
        if (last) mma_commit(bar_run_full + 8 * ra);
      }
      // no MMA may still write an accumulator when TMEM is freed
      mma_commit(bar_done);
      mbar_drain(bar_done, 0);
    }
  } else if (warp >= CONV_WARP0) {
    // ------------------------------------------------------ converters + sums
    const int ct = threadIdx.x - CONV_WARP0 * 32;  // time row of X this thread builds
    const int q = warp - CONV_WARP0;                // TMEM lane quarter (= rows 32q..)
    const float *xb = x + (size_t)b * Cin * T;
    float sum[NT];  // time sample t0 + ct, channels o0 .. o0 + NT - 1: FP32 run sums
#pragma unroll
    for (int e = 0; e < NT; ++e) sum[e] = 0.0f;
    // After this warp's first failed wait it does no more work and arrives on
    // nothing, but keeps walking the chunks so that the four converter warps
    // take the same named-barrier steps.
    bool dead = false;

    // stage x block blk (channels [CB blk, CB blk + CB)) into xs[blk & 1];
    // channels >= Cin and times outside [0, T) read as zero
    auto stage_x = [&](int blk) {
      float *dst = xs + (blk & 1) * CB * XW;
      const int i0 = blk * CB;
      const int width = BM + halo;
      for (int idx = ct; idx < CB * width; idx += NCONV) {
        const int ci = idx / width, n = idx - ci * width;
        const int i = i0 + ci, t = xt0 + n;
        const bool valid = (i < Cin) && (t >= 0) && (t < T);
        const float *src = valid ? xb + (size_t)i * T + t : xb;
        cp_async4_zfill(dst + ci * XW + n, src, valid);
      }
      cp_async_commit();
    };
    // add finished run p into the sums and hand its accumulator back
    auto promote = [&](int p) {
      const int ra = p & 1;
      if (dead || !warp_wait(bar_run_full + 8 * ra, (p >> 1) & 1, wc, 105)) {
        dead = true;
        return;
      }
      asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
#pragma unroll
      for (int c0 = 0; c0 < NT; c0 += 16) {
        uint32_t v[16];
        const unsigned taddr = tmem + ((unsigned)(32 * q) << 16) + (unsigned)(ra * MAX_NT + c0);
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
            "%13,%14,%15}, [%16];\n"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
              "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
              "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr)
            : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
        for (int e = 0; e < 16; ++e) sum[c0 + e] += __uint_as_float(v[e]);
      }
      asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_run_free + 8 * ra);
    };

    stage_x(0);
    int ready_blk = -1;
    int promoted = 0;  // runs added so far
    for (int c = 0; c < n_chunks; ++c) {
      const int s = c % NSTAGE, u = c / NSTAGE;
      const int sr = c % NRAW;
      const int kk0 = c * BK;
      // x blocks hold CB channels = CB K kk, a multiple of BK: a chunk never
      // straddles two blocks
      const int blk = (kk0 / K) / CB;
      const int m = c - blk * K;  // chunk index inside the block
      if (blk > ready_blk) {
        cp_async_wait_all();
        conv_bar_sync();  // everyone's copies of this block landed; the old block is free
        ready_blk = blk;
        if (!dead && (blk + 1) * CB < Cin) stage_x(blk + 1);
      }
      if (!dead && u > 0 && !warp_wait(bar_empty + 8 * s, (u - 1) & 1, wc, 103)) dead = true;
      if (!PRESPLIT && !dead && !warp_wait(bar_full_w + 8 * sr, (c / NRAW) & 1, wc, 104))
        dead = true;
      if (dead) continue;
      if (!PRESPLIT) {
      // W: split into hi and lo (elementwise over the swizzled tile)
      const unsigned char *w_raw = smem + WL::raw(sr);
      unsigned char *w_hi = smem + WL::hi(s);
      unsigned char *w_lo = smem + WL::lo(s);
      constexpr int WCH = W_BYTES / 16;  // 16-byte chunks of the weight tile
      constexpr int WPT = (WCH + NCONV - 1) / NCONV;
      float4 wv[WPT];
#pragma unroll
      for (int rr = 0; rr < WPT; ++rr)
        if (ct + rr * NCONV < WCH)
          wv[rr] = *reinterpret_cast<const float4 *>(w_raw + (ct + rr * NCONV) * 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_raw_free + 8 * sr);  // the TMA may refill the slot
#pragma unroll
      for (int rr = 0; rr < WPT; ++rr) {
        if (ct + rr * NCONV < WCH) {
          const int qo = (ct + rr * NCONV) * 16;
          const float4 v = wv[rr];
          const float4 h =
              make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
          *reinterpret_cast<float4 *>(w_hi + qo) = h;
          *reinterpret_cast<float4 *>(w_lo + qo) =
              make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
        }
      }
      }
      // X: time row ct of the im2col chunk, block-local kk = 32 m .. 32 m + 31
      unsigned char *x_hi = smem + OFF_XHI + s * X_TILE;
      unsigned char *x_lo = smem + OFF_XLO + s * X_TILE;
      const float *xrow = xs + (blk & 1) * CB * XW + ct;
      const int *offs = xoff + m * BK;
      float xv[BK];
#pragma unroll
      for (int e = 0; e < BK; e += 4) {
        const int4 o4 = *reinterpret_cast<const int4 *>(offs + e);
        xv[e] = xrow[o4.x];
        xv[e + 1] = xrow[o4.y];
        xv[e + 2] = xrow[o4.z];
        xv[e + 3] = xrow[o4.w];
      }
#pragma unroll
      for (int qq = 0; qq < BK / 4; ++qq) {
        float hv[4], lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hv[e] = tf32_hi(xv[4 * qq + e]);
          lv[e] = xv[4 * qq + e] - hv[e];
        }
        const int off = sw128_off(ct, 4 * qq);
        *reinterpret_cast<float4 *>(x_hi + off) = make_float4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<float4 *>(x_lo + off) = make_float4(lv[0], lv[1], lv[2], lv[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_ready + 8 * s);
      // a run whose MMAs were issued two chunks ago is complete by now
      if (c >= (promoted + 1) * RUN + 1) promote(promoted++);
    }
    cp_async_wait_all();
    while (!dead && promoted < n_runs) promote(promoted++);

    // ------------------------------------------------------------- epilogue
    // one thread per time sample: for each channel, the warp's 32 lanes touch
    // 32 consecutive samples of that channel's row (every stride-th sample for
    // a transposed-conv phase)
    const int t = t0 + ct;
    const int p = om.stride * t + om.offset + phase;
    if (!ctl.abort && t < y_len && p >= 0 && p < om.len) {
      // 16 channels at a time: the group's reads, then its writes
      const size_t base = (size_t)b * Cout * y_pitch + p;
#pragma unroll
      for (int g = 0; g < NT; g += 16) {
        float bb[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) bb[q] = bias_s[g + q];
        epi_group<16>(sum + g, bb, ep, y, base + (size_t)(o0 + g) * y_pitch, (size_t)y_pitch,
                      Cout - (o0 + g));
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();  // the MMA issuer has seen its final commit complete
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "n"(TMEM_COLS)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no
// link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// Channels per CTA: split Cout into the fewest tiles of at most 128 and round
// each to a multiple of 16 (the UMMA N granularity for M = 128).
int pick_nt(int Cout) {
  const int tiles = (Cout + MAX_NT - 1) / MAX_NT;
  const int per = (Cout + tiles - 1) / tiles;
  return (per + 15) / 16 * 16;
}

// Channels per CTA pair: the fewest tiles of at most 128, each a multiple of
// 32 (two halves of 16 rows, the smallest B half the pair's MMA takes).
int pick_nt_pair(int Cout) {
  const int tiles = (Cout + MAX_NT - 1) / MAX_NT;
  const int per = (Cout + tiles - 1) / tiles;
  return (per + 31) / 32 * 32;
}

template <int NT, bool PRESPLIT>
bv_status run_tc(const CUtensorMap &tmap, const CUtensorMap &tmap_lo, const float *x, int B,
                 int Cin, int T, const float *bias, int Cout, int K, int dil, int pad,
                 const Epi &ep, float *y, int y_len, int y_pitch, const OutMap &om,
                 cudaStream_t st) {
  BV_TRY(ensure_dynamic_smem((const void *)conv1d_tc_kernel<NT, PRESPLIT>, SMEM_BYTES,
                             "conv1d_tc smem attribute"));
  dim3 grid((y_len + BM - 1) / BM, (Cout + NT - 1) / NT, B * om.phases);
  if (grid.y > 65535 || grid.z > 65535) return fail(BV_ERR_SHAPE, "conv1d_tc: grid too large");
  conv1d_tc_kernel<NT, PRESPLIT><<<grid, THREADS, SMEM_BYTES, st>>>(
      tmap, tmap_lo, x, bias, y, Cin, T, Cout, K, dil, pad, y_len, y_pitch, ep, om,
      device_status_ptr(), wait_limit());
  return BV_OK;
}

// ---------------------------------------------------------------------------
// Time-major variant on CTA pairs.  The input arrives as two [B, T, Cin]
// planes, X_hi = tf32(x) and X_lo = x - X_hi (written by
// launch_transpose_split or the time-major activation), and the weights as
// tap-major [Cout, K Cin] hi / lo matrices, W'[o, j Cin + i] = w[o, i, j].
// With F16 the same holds with fp16 parts (X_hi = fp16(x), X_lo = fp16(x -
// X_hi); the weights' parts are of 2^12 W, scaled back in the run sums), a
// 128-byte operand row holds 64 channels instead of 32, and the MMAs are
// kind::f16 (K = 16) over the same 32-byte steps: the box geometry, swizzle,
// descriptors and barriers are those of tf32.
//
// Two CTAs of a cluster share each MMA (tcgen05 cta_group::2, M = 256): CTA r
// of the pair owns time rows t0 + 128 r .. + 127 (its half of the A operand
// and of the accumulator) and loads weight rows o0 + r NT/2 .. + NT/2 - 1
// (its half of the B operand), so each SM fetches half the weight bytes a
// lone CTA would; the weights are what every time tile re-reads from L2.
//
// For each 32-channel (fp16: 64-channel) block cb, one TMA box per plane brings input rows
// t0 - pad .. t0 - pad + 127 + (K - 1) d (zero outside [0, T), the conv's
// zero padding) by the block's 32 channels: K-major rows of 128 bytes, the A
// operand layout.  Tap j's A operand is the same box seen from row j d on:
// its descriptor starts j d rows in.  Both the TMA write and the tensor core's
// read place a 16-byte chunk by the absolute shared-memory address (chunk
// bits XOR row bits 7-9), so a start inside an 8-row group needs no base
// offset (measured on B200: setting the descriptor's base-offset field to the
// row phase breaks the result).  The input is fetched once per channel block;
// only the weight chunks (j, cb) stream through a ring.
//
// Roles: in each CTA one thread of warp 0 issues the weight loads and one of
// warp 2 the x loads, completing on the even CTA's barriers (which expect both
// CTAs' bytes); one thread of the even CTA issues the MMAs and commits to
// barriers in both CTAs; four warps per CTA add finished runs into FP32
// registers and write that CTA's rows of the [B, Cout, T] output with the
// usual epilogue.  A chunk is TAPS taps of one channel block (12 TAPS MMAs), so
// the per-chunk cost of a barrier wait and a commit in the issuing thread is
// spread over twice the tensor work.
constexpr int TM_MAX_HALO = 56;                       // (K - 1) d the x box can hold
// One CTA's half of a weight plane of an NT-channel tile: NT / 2 rows of 32
// channels (8 KB at NT = 128).
__host__ __device__ constexpr int tm_w_plane(int nt) { return (nt / 2) * BK * 4; }
// A weight chunk holds TAPS taps (hi and lo planes each); runs are 4 taps of
// 32 channels (128 kk) at 128 channels, 8 taps (256 kk) for narrower tiles,
// whatever the chunk size, so that the tensor core's truncating accumulation
// stays short (measured below).  Four-tap chunks
// for convs of three or more taps (half the barrier waits and commits per
// MMA: the [8, 384, 10006] K 7 layer 0.745 -> 0.661 ms); two-tap chunks, and
// so a deeper ring, for shorter ones (the transposed convs' phase convs).
__host__ __device__ constexpr int tm_w_slot(int taps, int nt) { return taps * 2 * tm_w_plane(nt); }
// Chunks per run: 128 kk at 128 channels; 256 kk for narrower tiles, whose
// runs are short against the sum warps' fixed cost per run (TMEM reads, the
// arrive).
__host__ __device__ constexpr int tm_run(int taps, int nt) { return (nt < MAX_NT ? 8 : 4) / taps; }
constexpr int TM_MAX_WSLOTS = 6;
constexpr int TM_BUDGET = 225 * 1024;                 // operand rings + barriers
constexpr int TM_SMEM_BYTES = TM_BUDGET + 1024;       // room to align the base
// x blocks in flight: two for 128-channel tiles (their weight chunks fill the
// rest), up to four for narrower tiles, whose few chunks per tile leave the
// x stream only a block or two of lead with two.
constexpr int TM_MAX_XSLOTS = 4;
// Run accumulators in TMEM (MAX_NT columns each; all 512 columns: the kernel
// is alone on its SM, its shared memory leaves room for no other CTA).  With
// four the issuer can run three runs ahead of the sum warps, which covers a
// tile's output loop.
constexpr int TM_ACC = 4;
constexpr int TM_TMEM_COLS = TM_ACC * MAX_NT;
static_assert(TM_TMEM_COLS <= 512 && (TM_ACC & (TM_ACC - 1)) == 0, "TMEM accumulators");
constexpr int TM_NBARS = 2 * TM_MAX_XSLOTS + 2 * TM_MAX_WSLOTS + 2 * TM_ACC + 1;
static_assert(TM_SMEM_BYTES + 1024 <= 227 * 1024, "shared memory budget");

// Output staging for the bulk-tensor stores of the output loop: per sum
// warp two buffers of 16 channels x 32 time steps.
constexpr int TM_STG_BUF = 16 * 32 * 4;
constexpr int TM_STG_BYTES = (NCONV / 32) * 2 * TM_STG_BUF;  // 16 KB
// Bytes of one x plane slot for `rows` rows (whole 1024-byte swizzle atoms).
__host__ __device__ constexpr int tm_x_plane(int rows) { return (rows * 128 + 1023) / 1024 * 1024; }
// Weight ring slots of `taps`-tap chunks of an NT-channel tile that fit
// beside xs x slots of `rows` rows and `stg` bytes of output staging.
__host__ __device__ constexpr int tm_w_slots(int rows, int taps, int nt, int stg, int xs) {
  return (TM_BUDGET - TM_NBARS * 8 - 2 * xs * tm_x_plane(rows) - stg) / tm_w_slot(taps, nt) <
                 TM_MAX_WSLOTS
             ? (TM_BUDGET - TM_NBARS * 8 - 2 * xs * tm_x_plane(rows) - stg) / tm_w_slot(taps, nt)
             : TM_MAX_WSLOTS;
}
// The ring depth the issuer needs: two four-tap or four two-tap chunks.
__host__ __device__ constexpr int tm_min_wslots(int taps) { return taps == 4 ? 2 : 4; }
// x slots of the layout: two at 128 channels, else the most (up to four) that
// leave the weight ring its depth.
__host__ __device__ constexpr int tm_x_slots(int rows, int taps, int nt, int stg) {
  return nt < MAX_NT && tm_w_slots(rows, taps, nt, stg, 4) >= tm_min_wslots(taps)   ? 4
         : nt < MAX_NT && tm_w_slots(rows, taps, nt, stg, 3) >= tm_min_wslots(taps) ? 3
                                                                                     : 2;
}
static_assert(tm_w_slots(BM + TM_MAX_HALO, 2, MAX_NT, 0, 2) >= tm_min_wslots(2) &&
                  tm_w_slots(BM + TM_MAX_HALO, 4, MAX_NT, 0, 2) >= tm_min_wslots(4),
              "weight ring depth");
static_assert(2 * 2 * tm_x_plane(BM + TM_MAX_HALO) + 2 * tm_w_slot(4, MAX_NT) + TM_NBARS * 8 <=
                  TM_BUDGET,
              "shared memory layout");
// Below 128 channels the staging always fits beside a full ring.
static_assert(tm_w_slots(BM + TM_MAX_HALO, 4, 96, TM_STG_BYTES, 2) >= tm_min_wslots(4) &&
                  tm_w_slots(BM + TM_MAX_HALO, 2, 96, TM_STG_BYTES, 2) >= tm_min_wslots(2),
              "ring depth with output staging");

// Instruction descriptor for the pair: D f32, A and B tf32, K-major, M = 256.
__host__ __device__ constexpr uint32_t make_idesc_pair(int nt) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(nt >> 3) << 17) |
         ((uint32_t)(256 >> 4) << 24);
}
// The same for kind::f16 with A and B fp16 (format 0).
__host__ __device__ constexpr uint32_t make_idesc_pair_f16(int nt) {
  return (1u << 4) | ((uint32_t)(nt >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::
                   : "memory");
}
// Shared::cluster address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ unsigned map_to_rank(unsigned addr, unsigned rank) {
  unsigned r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Relaxed: the arrive publishes no data of this thread's.  Its one use says
// that this thread's TMEM reads of a run accumulator are complete
// (tcgen05.wait::ld returned their values, then tcgen05.fence::before_thread_sync),
// so the MMA issuer may overwrite it; a release would also wait for this
// thread's outstanding global loads and stores (the residual prefetch, the
// previous tile's output), about a thousand cycles per run.
__device__ __forceinline__ void mbar_arrive_remote(unsigned cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr)
               : "memory");
}
// TMA loads of the pair: the destination is this CTA's shared memory, the
// completion goes to the even CTA's barrier (peer bit cleared).
constexpr unsigned kPeerBitMask = 0xFEFFFFFFu;
__device__ __forceinline__ void tma_load_3d_pair(unsigned dst, const CUtensorMap *map, int c0, int c1,
                                                 int c2, unsigned bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar & kPeerBitMask)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(unsigned dst, const CUtensorMap *map, int c0, int c1,
                                                 unsigned bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar & kPeerBitMask)
      : "memory");
}
// The A-collector qualifier: FILL keeps this MMA's A operand in the
// collector buffer, LASTUSE takes A from there (the same descriptor) and frees
// it, NONE reads A afresh.  Reusing A saves the tensor core one operand read.
enum class ACol { NONE, FILL, LASTUSE };
#define BV_MMA_PAIR(KIND, COL)                                                              \
  asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"                               \
               " tcgen05.mma.cta_group::2.kind::" KIND COL " [%0], %1, %2, %3, p;\n}\n" ::"r"( \
                   tmem_d),                                                                 \
               "l"(a), "l"(b), "r"(idesc), "r"(acc)                                         \
               : "memory")
// kind::tf32, or kind::f16 (A and B fp16) with F16.
template <ACol C, bool F16 = false>
__device__ __forceinline__ void mma_split_pair(unsigned tmem_d, uint64_t a, uint64_t b,
                                              uint32_t idesc, unsigned acc) {
  if constexpr (F16) {
    if constexpr (C == ACol::FILL) BV_MMA_PAIR("f16", ".collector::a::fill");
    else if constexpr (C == ACol::LASTUSE) BV_MMA_PAIR("f16", ".collector::a::lastuse");
    else BV_MMA_PAIR("f16", "");
  } else {
    if constexpr (C == ACol::FILL) BV_MMA_PAIR("tf32", ".collector::a::fill");
    else if constexpr (C == ACol::LASTUSE) BV_MMA_PAIR("tf32", ".collector::a::lastuse");
    else BV_MMA_PAIR("tf32", "");
  }
}
#undef BV_MMA_PAIR
// Arrive on the barrier at this offset in both CTAs once the MMAs issued so
// far have completed.
__device__ __forceinline__ void mma_commit_pair(unsigned bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n" ::"r"(bar),
      "h"((unsigned short)3)
      : "memory");
}

// Bulk-tensor store of a staged box (this CTA's shared memory -> global),
// tracked per thread in bulk groups.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, unsigned src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];\n" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
}
// At most N of this thread's bulk groups still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;\n" ::"n"(N) : "memory");
}
// Every bulk group of this thread complete (its writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}
// Generic-proxy writes to shared memory made visible to the bulk copies.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

template <int NT, int TAPS, bool STG, bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
conv1d_tm_kernel(const __grid_constant__ CUtensorMap tmap_xhi,
                 const __grid_constant__ CUtensorMap tmap_xlo,
                 const __grid_constant__ CUtensorMap tmap_whi,
                 const __grid_constant__ CUtensorMap tmap_wlo,
                 const __grid_constant__ CUtensorMap tmap_y, const float *__restrict__ bias,
                 float *y, int Cin, int Cout, int K, int dil, int pad, int y_len, int y_pitch,
                 Epi ep, OutMap om, int *status, long long wait_limit, int tpairs, int ntiles,
                 int n_tiles) {
  static_assert(NT % 32 == 0 && NT >= 32 && NT <= MAX_NT, "UMMA N for M = 256, halves of 16");
  constexpr uint32_t IDESC = F16 ? make_idesc_pair_f16(NT) : make_idesc_pair(NT);
  // channels per block: one 128-byte operand row (32 tf32 or 64 fp16 values;
  // an MMA takes 32 bytes of it, K = 8 or 16)
  constexpr int CB = F16 ? 2 * BK : BK;
  constexpr unsigned W_TX_TAP = 2u * 2u * (NT / 2) * BK * 4;  // one tap: both CTAs, hi and lo
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ Ctl ctl;
  const unsigned rank = cluster_rank();
  const bool leader = (rank == 0);
  const int xrows = BM + (K - 1) * dil;  // rows of one x box
  const int XP = tm_x_plane(xrows);
  static_assert(TAPS == 2 || TAPS == 4, "taps per weight chunk");
  constexpr int TM_W_PLANE = tm_w_plane(NT);
  constexpr int TM_W_SLOT = tm_w_slot(TAPS, NT), TM_RUN = tm_run(TAPS, NT);
  // STG: the output loop stages each 16-channel group in shared memory and
  // writes it with one bulk-tensor store through tmap_y (plain [B, Cout,
  // y_pitch] outputs whose rows start on 16 bytes; the launcher checked that
  // the staging leaves the ring its depth)
  const int XS = tm_x_slots(xrows, TAPS, NT, STG ? TM_STG_BYTES : 0);
  const int NW = tm_w_slots(xrows, TAPS, NT, STG ? TM_STG_BYTES : 0, XS);
  const unsigned X_TX = 2u * 2u * (unsigned)xrows * 128u;  // both CTAs, hi and lo
  unsigned char *wbase = smem + 2 * XS * XP;
  unsigned char *stg_base = wbase + NW * TM_W_SLOT;  // 1024-byte aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(stg_base + (STG ? TM_STG_BYTES : 0));
  // barriers (the leader's full and run-free barriers serve the pair):
  // x block loaded / consumed (XS slots), weight chunk loaded / consumed
  // (NW slots), run accumulated / run accumulator read (2), every MMA done
  const unsigned bar_xfull = smem_u32(&bars[0]);
  const unsigned bar_xempty = smem_u32(&bars[TM_MAX_XSLOTS]);
  const unsigned bar_wfull = smem_u32(&bars[2 * TM_MAX_XSLOTS]);
  const unsigned bar_wempty = smem_u32(&bars[2 * TM_MAX_XSLOTS + TM_MAX_WSLOTS]);
  const unsigned bar_run_full = smem_u32(&bars[2 * TM_MAX_XSLOTS + 2 * TM_MAX_WSLOTS]);
  const unsigned bar_run_free =
      smem_u32(&bars[2 * TM_MAX_XSLOTS + 2 * TM_MAX_WSLOTS + TM_ACC]);
  const unsigned bar_done = smem_u32(&bars[2 * TM_MAX_XSLOTS + 2 * TM_MAX_WSLOTS + 2 * TM_ACC]);
  // x slot s, plane (0 hi, 1 lo); weight slot s, tap t of the chunk, plane
  auto x_at = [&](int slot, int plane) { return smem_u32(smem + (2 * slot + plane) * XP); };
  auto w_at = [&](int slot, int tap, int plane) {
    return smem_u32(wbase + slot * TM_W_SLOT + (2 * tap + plane) * TM_W_PLANE);
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The pair walks the tiles cid, cid + P, ... (P pairs in the grid); tile
  // tau is time pair tau % tpairs, output-channel tile (tau / tpairs) %
  // ntiles and row-phase bz = tau / (tpairs ntiles).  Every role of both CTAs
  // walks the same tiles, and the ring, run and phase counters run on across
  // tiles, so the producers fill the next tile's operands and the MMAs start
  // on it while the sum warps write the previous one out.
  const int cid = (int)(blockIdx.x >> 1), P = (int)(gridDim.x >> 1);
  struct Tile {
    int t0, o0, b, phase;
  };
  auto tile_of = [&](int tau) {
    Tile tl;
    const int tp = tau % tpairs, rest = tau / tpairs;
    const int bz = rest / ntiles;
    tl.t0 = tp * (2 * BM) + (int)rank * BM;  // this CTA's rows
    tl.o0 = (rest - bz * ntiles) * NT;
    tl.b = bz / om.phases;
    tl.phase = bz - tl.b * om.phases;  // weight rows phase Cout .., output offset + phase
    return tl;
  };
  const int n_cb = (Cin + CB - 1) / CB;  // channel blocks (channels past Cin read as 0)
  const int Cpad = n_cb * CB;            // weight row stride per tap
  const int n_tc = (K + TAPS - 1) / TAPS;  // chunks per block: taps 0 .. TAPS - 1, ...
  const int n_chunks = n_cb * n_tc;
  const int n_runs = (n_chunks + TM_RUN - 1) / TM_RUN;  // per tile
  // a wait that runs out marks both CTAs of the pair aborted
  const WaitCtx wc{&ctl, map_to_rank(smem_u32(&ctl.abort), rank ^ 1u), status, wait_limit};

  if (threadIdx.x == 0) {
    ctl.abort = 0;
    mbar_init(bar_done, 1);
    for (int s = 0; s < XS; ++s) {
      mbar_init(bar_xfull + 8 * s, 1);
      mbar_init(bar_xempty + 8 * s, 1);
    }
    for (int s = 0; s < TM_ACC; ++s) {
      mbar_init(bar_run_full + 8 * s, 1);
      mbar_init(bar_run_free + 8 * s, 2 * NCONV / 32);  // sum warps of both CTAs
    }
    for (int s = 0; s < NW; ++s) {
      mbar_init(bar_wfull + 8 * s, 1);
      mbar_init(bar_wempty + 8 * s, 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&ctl.tmem)),
                 "n"(TM_TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  cluster_sync();  // both CTAs' barriers exist before anyone signals them
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const unsigned tmem = ctl.tmem;

  if (warp == 2) {
    // ---------------------------------------------------- TMA producer: x blocks
    // (a thread of its own, so a block waiting for its slot never holds up
    // the weight stream)
    if (lane == 0) {
      // a failed wait stops the loads; a slot holds at most one load not yet
      // seen complete, the last one issued into it (gcb counts the blocks
      // issued over all tiles)
      int gcb = 0, xs = 0, xu = 0;  // slot xs of pass xu over the x ring
      bool ok = true;
      for (int tau = cid; tau < n_tiles && ok; tau += P) {
        const Tile tl = tile_of(tau);
        for (int cb = 0; cb < n_cb; ++cb) {
          if (xu > 0 && !mbar_wait(bar_xempty + 8 * xs, (xu - 1) & 1, wc, 111)) {
            ok = false;
            break;
          }
          const unsigned fb = bar_xfull + 8 * xs;
          if (leader) mbar_arrive_tx(fb, X_TX);
          tma_load_3d_pair(x_at(xs, 0), &tmap_xhi, cb * CB, tl.t0 - pad, tl.b, fb);
          tma_load_3d_pair(x_at(xs, 1), &tmap_xlo, cb * CB, tl.t0 - pad, tl.b, fb);
          ++gcb;
          if (++xs == XS) {
            xs = 0;
            ++xu;
          }
        }
      }
      if (leader)
        for (int c = gcb - XS; c < gcb; ++c)
          if (c >= 0) mbar_drain(bar_xfull + 8 * (c % XS), (c / XS) & 1);
    }
  } else if (warp == 0) {
    // ----------------------------------------------- TMA producer: weight chunks
    if (lane == 0) {
      // slot ws of pass wu over the ring (counters, not divisions: this loop
      // and the MMA issuer's are single threads on the critical path)
      int ws = 0, wu = 0, gc = 0;  // gc: chunks issued over all tiles
      bool ok = true;
      for (int tau = cid; tau < n_tiles && ok; tau += P) {
        const Tile tl = tile_of(tau);
        const int row = tl.phase * Cout + tl.o0 + (int)rank * (NT / 2);
        for (int cb = 0; cb < n_cb && ok; ++cb) {
          for (int q = 0; q < n_tc; ++q) {
            if (wu > 0 && !mbar_wait(bar_wempty + 8 * ws, (wu - 1) & 1, wc, 112)) {
              ok = false;
              break;
            }
            const int j0 = TAPS * q, ntap = (K - j0) < TAPS ? (K - j0) : TAPS;
            const unsigned fb = bar_wfull + 8 * ws;
            if (leader) mbar_arrive_tx(fb, W_TX_TAP * ntap);
            for (int t = 0; t < ntap; ++t) {
              const int col = (j0 + t) * Cpad + cb * CB;
              tma_load_2d_pair(w_at(ws, t, 0), &tmap_whi, col, row, fb);
              tma_load_2d_pair(w_at(ws, t, 1), &tmap_wlo, col, row, fb);
            }
            ++gc;
            if (++ws == NW) {
              ws = 0;
              ++wu;
            }
          }
        }
      }
      // drain: the pair's last loads land before the leader can exit (the
      // leader's full barriers count the odd CTA's bytes too, and the final
      // cluster barrier holds the odd CTA until then)
      if (leader)
        for (int c = gc - NW; c < gc; ++c)
          if (c >= 0) mbar_drain(bar_wfull + 8 * (c % NW), (c / NW) & 1);
    }
  } else if (warp == 1) {
    // ----------------------------------------------- MMA issuer (leader only)
    if (leader && lane == 0) {
      // descriptors are formed once per operand tile and advanced by adding
      // the byte offset / 16 (the start-address field; shared addresses stay
      // below 256 KB, so the field never carries).  xs / ws: the x and
      // weight ring slots with their phases; gr: runs issued over all
      // tiles (a run never spans two tiles).
      int gr = 0, ws = 0, xs = 0;
      unsigned wphase = 0, xphase = 0;
      bool ok = true;
      for (int tau = cid; tau < n_tiles && ok; tau += P) {
        int c = 0;  // chunk within the tile
        for (int cb = 0; cb < n_cb && ok; ++cb) {
          if (!mbar_wait(bar_xfull + 8 * xs, xphase, wc, 113)) {
            ok = false;
            break;
          }
          const uint64_t dxh = sw128_desc(x_at(xs, 0)), dxl = sw128_desc(x_at(xs, 1));
          for (int q = 0; q < n_tc; ++q, ++c) {
            const int ra = gr & (TM_ACC - 1);
            const bool first = (c % TM_RUN) == 0;
            const bool last = (c % TM_RUN) == TM_RUN - 1 || c == n_chunks - 1;
            // both CTAs' sum warps have read this accumulator's run gr - TM_ACC
            if ((first && gr >= TM_ACC &&
                 !mbar_wait(bar_run_free + 8 * ra, ((gr / TM_ACC) - 1) & 1, wc, 114)) ||
                !mbar_wait(bar_wfull + 8 * ws, wphase, wc, 115)) {
              ok = false;
              break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
            const unsigned acc = tmem + (unsigned)(ra * MAX_NT);
            const int j0 = TAPS * q, ntap = (K - j0) < TAPS ? (K - j0) : TAPS;
            for (int t = 0; t < ntap; ++t) {
              const uint64_t rows = (uint64_t)((j0 + t) * dil * 8);  // tap's first row, in 16 B
              const uint64_t ah = dxh + rows, al = dxl + rows;
              const uint64_t bh = sw128_desc(w_at(ws, t, 0)), bl = sw128_desc(w_at(ws, t, 1));
#pragma unroll
              for (int k = 0; k < BK / 8; ++k) {  // 8 tf32 or 16 fp16 = 32 B = 2 x 16 B per MMA
                const uint64_t o = 2 * k;
                // X_hi is the A operand of two products: read it once
                mma_split_pair<ACol::FILL, F16>(acc, ah + o, bh + o, IDESC,
                                               (first && t == 0 && k == 0) ? 0u : 1u);
                mma_split_pair<ACol::LASTUSE, F16>(acc, ah + o, bl + o, IDESC, 1u);
                mma_split_pair<ACol::NONE, F16>(acc, al + o, bh + o, IDESC, 1u);
              }
            }
            mma_commit_pair(bar_wempty + 8 * ws);  // both CTAs may refill the weight slot
            if (q == n_tc - 1) mma_commit_pair(bar_xempty + 8 * xs);  // and the x slot
            if (last) {
              mma_commit_pair(bar_run_full + 8 * ra);
              ++gr;
            }
            if (++ws == NW) {
              ws = 0;
              wphase ^= 1u;
            }
          }
          if (++xs == XS) {
            xs = 0;
            xphase ^= 1u;
          }
        }
      }
      // every MMA issued above has completed before TMEM can be freed
      mma_commit_pair(bar_done);
      mbar_drain(bar_done, 0);
    }
  } else if (warp >= CONV_WARP0) {
    // ------------------------------------------------------ run sums + output
    const int ct = threadIdx.x - CONV_WARP0 * 32;  // time row of this thread
    const int q = warp - CONV_WARP0;                // TMEM lane quarter (= rows 32q..)
    const unsigned run_free_leader = map_to_rank(bar_run_free, 0);
    constexpr int NG = NT / 16;                // 16-channel groups of a tile
    constexpr int FOLD_G = NT < MAX_NT ? 3 : 1;  // residual groups folded per run
    int gr = 0;   // runs read over all tiles
    int sgi = 0;  // staged output groups of this warp over all tiles
    bool alive = true;
    for (int tau = cid; tau < n_tiles && alive; tau += P) {
      const Tile tl = tile_of(tau);
      // this tile's biases, loaded before its runs so that the load latency
      // hides behind the run waits: lane l holds channels o0 + l + 32 i,
      // handed to the 16-channel groups by shuffles in the output loop
      float breg[NT / 32];
#pragma unroll
      for (int i = 0; i < NT / 32; ++i) {
        const int o = tl.o0 + lane + 32 * i;
        breg[i] = (bias && o < Cout) ? __ldg(bias + o) : 0.0f;
      }
      float sum[NT];
#pragma unroll
      for (int e = 0; e < NT; ++e) sum[e] = 0.0f;
      // The residual of this thread's output row, FOLD_G groups of 16
      // channels per run for the first runs: a run's loads are issued before
      // its wait, so their latency hides behind it instead of the output loop,
      // and the values join the sum after the run's arrive ((conv + residual)
      // + bias instead of (conv + bias) + residual).  Narrow tiles have few
      // runs per tile, so they fold three groups a run.
      const int t_out = tl.t0 + ct;
      const int p_out = om.stride * t_out + om.offset + tl.phase;  // output sample
      const bool in = t_out < y_len && p_out >= 0 && p_out < om.len;
      const size_t base = (size_t)tl.b * Cout * y_pitch + p_out;
      const bool fold = ep.residual != nullptr;
      for (int p = 0; p < n_runs; ++p, ++gr) {
        const int ra = gr & (TM_ACC - 1);
        const bool fold_p = fold && in && p * FOLD_G < NG;
        float r[16 * FOLD_G];
        if (fold_p) {
#pragma unroll
          for (int j = 0; j < FOLD_G; ++j) {
            const int g = p * FOLD_G + j;
            const int valid = g < NG ? Cout - (tl.o0 + 16 * g) : 0;
            const float *rp = ep.residual + base + (size_t)(tl.o0 + 16 * g) * y_pitch;
#pragma unroll
            for (int e = 0; e < 16; ++e)
              r[16 * j + e] = e < valid ? __ldg(rp + (size_t)e * y_pitch) : 0.0f;
          }
        }
        if (!warp_wait(bar_run_full + 8 * ra, (gr / TM_ACC) & 1, wc, 116)) {
          alive = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        // 32 columns per wait: two loads in flight
#pragma unroll
        for (int c0 = 0; c0 < NT; c0 += 32) {
          uint32_t v[32];
          const unsigned taddr = tmem + ((unsigned)(32 * q) << 16) + (unsigned)(ra * MAX_NT + c0);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,"
                "%12,%13,%14,%15}, [%16];\n"
                : "=r"(v[16 * h + 0]), "=r"(v[16 * h + 1]), "=r"(v[16 * h + 2]),
                  "=r"(v[16 * h + 3]), "=r"(v[16 * h + 4]), "=r"(v[16 * h + 5]),
                  "=r"(v[16 * h + 6]), "=r"(v[16 * h + 7]), "=r"(v[16 * h + 8]),
                  "=r"(v[16 * h + 9]), "=r"(v[16 * h + 10]), "=r"(v[16 * h + 11]),
                  "=r"(v[16 * h + 12]), "=r"(v[16 * h + 13]), "=r"(v[16 * h + 14]),
                  "=r"(v[16 * h + 15])
                : "r"(taddr + 16u * h)
                : "memory");
          asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
          // the fp16 weights carry kTmF16WScale (a power of two: exact)
          constexpr float kBack = F16 ? 1.0f / kTmF16WScale : 1.0f;
#pragma unroll
          for (int e = 0; e < 32; ++e) sum[c0 + e] = fmaf(__uint_as_float(v[e]), kBack, sum[c0 + e]);
        }
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(run_free_leader + 8 * ra);
        if (fold_p) {
#pragma unroll
          for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int j = 0; j < FOLD_G; ++j)
              if (g == p * FOLD_G + j) {
#pragma unroll
                for (int e = 0; e < 16; ++e) sum[16 * g + e] += r[16 * j + e];
              }
        }
      }
      if (!alive || ctl.abort) break;
#pragma unroll
      for (int g = 0; g < NT; g += 16) {
        float bb[16];  // every lane of the warp takes part in the shuffles
#pragma unroll
        for (int e = 0; e < 16; ++e) bb[e] = __shfl_sync(0xffffffffu, breg[(g + e) >> 5], (g + e) & 31);
        // 16 channels at a time: the group's reads, then its writes (without
        // the residual where it joined the sum above)
        Epi eg = ep;
        if (fold && g / 16 < n_runs * FOLD_G) eg.residual = nullptr;
        const size_t idx0 = base + (size_t)(tl.o0 + g) * y_pitch;
        if constexpr (STG) {
          // staged: the warp's 32 time steps x 16 channels go out in one
          // bulk store, which clips rows past y_len and channels past Cout
          float val[16];  // rows past y_len stage zeros (the store clips them)
#pragma unroll
          for (int e = 0; e < 16; ++e) val[e] = 0.0f;
          if (in) epi_values<16>(sum + g, bb, eg, y, idx0, (size_t)y_pitch, Cout - (tl.o0 + g), val);
          if (tl.o0 + g < Cout && tl.t0 + 32 * q < y_len) {  // warp-uniform
            float *sb = reinterpret_cast<float *>(stg_base + (2 * q + (sgi & 1)) * TM_STG_BUF);
            if (sgi >= 2) {  // the store that read this buffer two groups ago is done
              if (lane == 0) bulk_wait_read<1>();
              __syncwarp();
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) sb[32 * e + lane] = val[e];
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_3d(&tmap_y, smem_u32(sb), tl.t0 + 32 * q, tl.o0 + g, tl.b);
              bulk_commit();
            }
            ++sgi;
          }
        } else if (in) {
          epi_group<16>(sum + g, bb, eg, y, idx0, (size_t)y_pitch, Cout - (tl.o0 + g));
        }
      }
    }
    // the staged stores have written y before the kernel can end
    if (STG && lane == 0) bulk_wait_all();
    __syncwarp();
  }

  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  // After an abort the odd CTA may have loads in flight that the leader's
  // barriers did not count (issued after the leader stopped); they land in a
  // few microseconds, so it waits 64 us before it can exit.
  if (!leader && threadIdx.x == 0 && ctl.abort)
    for (int i = 0; i < 64; ++i) __nanosleep(1000);
  // every MMA of the pair has completed (the leader saw its final commit) and
  // every remote arrive has landed before either CTA frees TMEM or its
  // shared memory
  cluster_sync();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "n"(TM_TMEM_COLS)
                 : "memory");
  }
}

// CTA pairs that fit on the device at once (one CTA per SM).
int tm_pairs() {
  constexpr int kMaxDev = 64;
  static int cache[kMaxDev];
  int dev = 0;
  cudaGetDevice(&dev);
  const int slot = dev >= 0 && dev < kMaxDev ? dev : 0;
  int n = __atomic_load_n(&cache[slot], __ATOMIC_RELAXED);
  if (n == 0) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    n = sms / 2 > 0 ? sms / 2 : 1;
    __atomic_store_n(&cache[slot], n, __ATOMIC_RELAXED);
  }
  return n;
}

// Output tensor map for the staged output loop: y as [B, Cout, y_pitch]
// with y_len valid time steps, box 32 time steps x 16 channels.  Returns
// false (no staging) where the rows do not start on 16 bytes.
bool encode_y_tm(CUtensorMap *tmap, float *y, int B, int Cout, int y_len, int y_pitch) {
  if ((reinterpret_cast<uintptr_t>(y) & 15u) != 0 || y_pitch % 4 != 0 || y_len > y_pitch)
    return false;
  const cuuint64_t dims[3] = {(cuuint64_t)y_len, (cuuint64_t)Cout, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)y_pitch * sizeof(float),
                                 (cuuint64_t)y_pitch * Cout * sizeof(float)};
  const cuuint32_t box[3] = {32, 16, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, y, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int TAPS, bool F16>
bv_status run_tm(const CUtensorMap &xh, const CUtensorMap &xl, const CUtensorMap &wh,
                 const CUtensorMap &wl, int B, int Cin, const float *bias, int Cout, int K,
                 int dil, int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                 const OutMap &om, cudaStream_t st) {
  // Staged output loop for plain outputs (not the transposed convs' phase
  // interleave) when the staging leaves the weight ring its depth.
  CUtensorMap ym;
  const bool plain = om.stride == 1 && om.offset == 0 && om.phases == 1 && om.len == y_len;
  const bool stg = plain &&
                   tm_w_slots(BM + (K - 1) * dil, TAPS, NT, TM_STG_BYTES, 2) >= tm_min_wslots(TAPS) &&
                   encode_y_tm(&ym, y, B, Cout, y_len, y_pitch);
  if (!stg) std::memset(&ym, 0, sizeof(ym));
  const void *kern = stg ? (const void *)conv1d_tm_kernel<NT, TAPS, true, F16>
                         : (const void *)conv1d_tm_kernel<NT, TAPS, false, F16>;
  BV_TRY(ensure_dynamic_smem(kern, TM_SMEM_BYTES, "conv1d_tm smem attribute"));
  // persistent: at most one CTA pair per two SMs, each walking its share of
  // the (time pair, output-channel tile, row-phase) tiles
  const long long tpairs = (y_len + 2 * BM - 1) / (2 * BM), ntiles = (Cout + NT - 1) / NT;
  const long long n_tiles = tpairs * ntiles * (long long)B * om.phases;
  if (n_tiles > 0x7fffffffLL) return fail(BV_ERR_SHAPE, "conv1d_tm: too many tiles");
  const long long pairs = std::min<long long>(n_tiles, tm_pairs());
  if (stg)
    conv1d_tm_kernel<NT, TAPS, true, F16><<<dim3((unsigned)(2 * pairs)), THREADS, TM_SMEM_BYTES, st>>>(
        xh, xl, wh, wl, ym, bias, y, Cin, Cout, K, dil, pad, y_len, y_pitch, ep, om,
        device_status_ptr(), wait_limit(), (int)tpairs, (int)ntiles, (int)n_tiles);
  else
    conv1d_tm_kernel<NT, TAPS, false, F16><<<dim3((unsigned)(2 * pairs)), THREADS, TM_SMEM_BYTES, st>>>(
        xh, xl, wh, wl, ym, bias, y, Cin, Cout, K, dil, pad, y_len, y_pitch, ep, om,
        device_status_ptr(), wait_limit(), (int)tpairs, (int)ntiles, (int)n_tiles);
  return BV_OK;
}

// [B, T, C] plane as a 3-D tensor map, box of one 128-byte row (32 fp32 or
// 64 fp16 channels) x `rows` times.
bv_status encode_x_tm(CUtensorMap *tmap, const float *x, int B, int C, int T, int rows,
                      bool f16 = false) {
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0)
    return fail(BV_ERR_UNSUPPORTED, "conv1d_tm: input not 16-byte aligned");
  const cuuint64_t es = f16 ? 2 : 4;
  const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)T * C * es};
  const cuuint32_t box[3] = {f16 ? 2u * BK : (cuuint32_t)BK, (cuuint32_t)rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encode_fn()(tmap, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           3, const_cast<float *>(x), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(BV_ERR_CUDA, "conv1d_tm: tensor map encode failed (%d)", (int)r);
  return BV_OK;
}

}  // namespace

// The tensor-core path pays a fixed cost per CTA (barriers, TMEM, pipeline
// fill) that narrow layers cannot amortise: measured on B200, the FP32 SIMT
// kernel is as fast or faster below about 40 output channels or 192 reduction
// terms (e.g. 12- and 24-channel stages, 48 channels with k = 3, and the
// 1-channel conv_post), and the tensor cores win from 48 channels with k >= 7.
bool conv1d_tc_supported(int Cin, int Cout, int K, int dil) {
  return Cout >= 40 && Cin * K >= 192 && K <= MAX_K && (Cin * K) % 4 == 0 &&
         (K - 1) * dil <= MAX_HALO && encode_fn() != nullptr;
}

namespace {

// Weight tensor map: [rows, Cin K] fp32 (fp16 with f16), box one 128-byte
// row x nt, 128-byte swizzle.
bv_status encode_w(CUtensorMap *tmap, const float *w, int rows, int KK, int nt, bool f16 = false) {
  if ((reinterpret_cast<uintptr_t>(w) & 15u) != 0)
    return fail(BV_ERR_UNSUPPORTED, "conv1d_tc: weights not 16-byte aligned");
  const cuuint64_t dims[2] = {(cuuint64_t)KK, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)KK * (f16 ? 2 : 4)};
  const cuuint32_t box[2] = {f16 ? 2u * BK : (cuuint32_t)BK, (cuuint32_t)nt};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = encode_fn()(tmap, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                           2, const_cast<float *>(w), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(BV_ERR_CUDA, "conv1d_tc: tensor map encode failed (%d)", (int)r);
  return BV_OK;
}

// Launch the NT instance.  w: the [w_rows, Cin K] weight matrix; or, when
// split is set, w holds tf32(W) followed by W - tf32(W) (each [w_rows, Cin K])
// and both operands go straight from global memory to the MMA, otherwise the
// kernel splits the raw weights itself.
bv_status launch_tc_impl(const char *cls, const float *x, int B, int Cin, int T, const float *w,
                         bool split, int w_rows, const float *bias, int Cout, int K, int dil,
                         int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                         const OutMap &om, double flops, double bytes, cudaStream_t st) {
  if (!encode_fn()) return fail(BV_ERR_UNSUPPORTED, "conv1d_tc: no cuTensorMapEncodeTiled");
  const int nt = pick_nt(Cout);
  CUtensorMap tmap, tmap_lo;
  bv_status s = encode_w(&tmap, w, w_rows, Cin * K, nt);
  if (s != BV_OK) return s;
  if (split) {
    s = encode_w(&tmap_lo, w + (size_t)w_rows * Cin * K, w_rows, Cin * K, nt);
    if (s != BV_OK) return s;
  } else {
    tmap_lo = tmap;
  }
  {
    LaunchTimer tm(st, cls, flops, bytes);
#define BV_TC_CASE(N)                                                                          \
  case N:                                                                                      \
    s = split ? run_tc<N, true>(tmap, tmap_lo, x, B, Cin, T, bias, Cout, K, dil, pad, ep, y,   \
                               y_len, y_pitch, om, st)                                         \
              : run_tc<N, false>(tmap, tmap_lo, x, B, Cin, T, bias, Cout, K, dil, pad, ep, y,  \
                                y_len, y_pitch, om, st);                                       \
    break;
    switch (nt) {
      BV_TC_CASE(16)
      BV_TC_CASE(32)
      BV_TC_CASE(48)
      BV_TC_CASE(64)
      BV_TC_CASE(80)
      BV_TC_CASE(96)
      BV_TC_CASE(112)
      BV_TC_CASE(128)
      default:
        return fail(BV_ERR_UNSUPPORTED, "conv1d_tc: tile %d", nt);
    }
#undef BV_TC_CASE
  }
  if (s != BV_OK) return s;
  count_launch();
  return check_launch("conv1d_tc_kernel");
}

// wp[r][o][i nt + j] = w[i][o][r + s (nt - 1 - j)] (zero past K): phase r of
// the transposed conv as an ordinary nt-tap conv over the input samples.
__global__ void convt_repack_kernel(const float *__restrict__ w, float *__restrict__ wp,
                                    float *__restrict__ wp_lo, int Cin, int Cout, int K, int S,
                                    int nt) {
  const long long total = (long long)S * Cout * Cin * nt;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(idx % nt);
    long long rest = idx / nt;
    const int i = (int)(rest % Cin);
    rest /= Cin;
    const int o = (int)(rest % Cout);
    const int r = (int)(rest / Cout);
    const int k = r + S * (nt - 1 - j);
    const float v = k < K ? w[((size_t)i * Cout + o) * K + k] : 0.0f;
    const float h = tf32_hi(v);
    wp[idx] = h;
    wp_lo[idx] = v - h;
  }
}

// Tap-major phase weights for the time-major kernel: wp[r][o][j cp + i] =
// w[i][o][r + S (nt - 1 - j)] split into tf32 hi / lo (zero past K or Cin).
// f16: the parts are fp16 of kTmF16WScale W (wp and wp_lo then hold halves)
__global__ void convt_repack_tm_kernel(const float *__restrict__ w, float *__restrict__ wp,
                                       float *__restrict__ wp_lo, int Cin, int Cout, int K, int S,
                                       int nt, int cp, int f16, int *status) {
  const long long total = (long long)S * Cout * nt * cp;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % cp);
    long long rest = idx / cp;
    const int j = (int)(rest % nt);
    rest /= nt;
    const int o = (int)(rest % Cout);
    const int r = (int)(rest / Cout);
    const int k = r + S * (nt - 1 - j);
    const float v = (k < K && i < Cin) ? w[((size_t)i * Cout + o) * K + k] : 0.0f;
    if (f16) {
      const float vs = v * kTmF16WScale;
      if (fabsf(vs) >= 65504.0f && status) atomicExch(status, kStatusF16Range);  // |W| >= 16
      const __half h = __float2half_rn(vs);
      reinterpret_cast<__half *>(wp)[idx] = h;
      reinterpret_cast<__half *>(wp_lo)[idx] = __float2half_rn(vs - __half2float(h));
    } else {
      const float h = tf32_hi(v);
      wp[idx] = h;
      wp_lo[idx] = v - h;
    }
  }
}

// dst[0 .. n) = tf32(src), dst[n .. 2n) = src - tf32(src), per table entry
// (float4 where the entry allows it; tap-major entries reorder as they go)
__global__ void split_weights_kernel(SplitTable tab, int *status) {
  for (int e = blockIdx.y; e < tab.n; e += gridDim.y) {
    const float *__restrict__ src = tab.src[e];
    float *__restrict__ hi = tab.dst[e];
    const long long n = tab.count[e];
    float *__restrict__ lo = hi + n;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) &&
                     ((reinterpret_cast<uintptr_t>(hi) & 15u) == 0);
    if (tab.cin[e] > 0) {
      // one output row o at a time, 64 input channels per pass: the slice
      // src[o][i0 .. i0 + 64)[0 .. k) is contiguous, and so is each tap's run
      // dst[o][j cp + i0 .. + 64); shared memory turns one into the other.
      // Rows are padded to cp = tm_cin_pad(cin) channels per tap with zeros
      // (tm_cin_pad_f16 for the fp16 split, whose hi and lo are halves).
      __shared__ float sl[64 * MAX_K];
      const bool f16 = tab.f16[e] != 0;
      const int cin = tab.cin[e], k = tab.k[e];
      const int cp = f16 ? tm_cin_pad_f16(cin) : tm_cin_pad(cin);
      const long long row = (long long)cin * k, drow = (long long)cp * k;
      const long long rows = n / row;
      lo = hi + rows * drow;
      __half *const hi16 = reinterpret_cast<__half *>(hi), *const lo16 = hi16 + rows * drow;
      for (long long o = blockIdx.x; o < rows; o += gridDim.x) {
        for (int i0 = 0; i0 < cin; i0 += 64) {
          const int ni = cin - i0 < 64 ? cin - i0 : 64;
          const float *sp = src + o * row + (long long)i0 * k;
          for (int q = threadIdx.x; q < ni * k; q += blockDim.x) sl[q] = sp[q];
          __syncthreads();
          for (int q = threadIdx.x; q < ni * k; q += blockDim.x) {
            const int j = q / ni, ii = q - j * ni;
            const long long d = o * drow + (long long)j * cp + i0 + ii;
            if (f16) {
              const float v = sl[ii * k + j] * kTmF16WScale;
              // fp16 holds |2^12 W| < 65504: a weight of 16 or more is reported
              if (fabsf(v) >= 65504.0f && status) atomicExch(status, kStatusF16Range);
              const __half h = __float2half_rn(v);
              hi16[d] = h;
              lo16[d] = __float2half_rn(v - __half2float(h));
            } else {
              const float v = sl[ii * k + j], h = tf32_hi(v);
              hi[d] = h;
              lo[d] = v - h;
            }
          }
          __syncthreads();
        }
        for (int q = threadIdx.x; q < (cp - cin) * k; q += blockDim.x) {
          const int j = q / (cp - cin), ii = cin + q - j * (cp - cin);
          const long long d = o * drow + (long long)j * cp + ii;
          if (f16) {
            hi16[d] = __float2half_rn(0.0f);
            lo16[d] = __float2half_rn(0.0f);
          } else {
            hi[d] = 0.0f;
            lo[d] = 0.0f;
          }
        }
      }
    } else if (vec) {
      for (long long i = i0; i < n / 4; i += stride) {
        const float4 v = reinterpret_cast<const float4 *>(src)[i];
        const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
        reinterpret_cast<float4 *>(hi)[i] = h;
        reinterpret_cast<float4 *>(lo)[i] = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
      }
    } else {
      for (long long i = i0; i < n; i += stride) {
        const float v = src[i], h = tf32_hi(v);
        hi[i] = h;
        lo[i] = v - h;
      }
    }
  }
}

// hi[b, t, c] = tf32(x[b, c, t]), lo = x - hi: 32 x 32 tiles through shared
// memory, reads along t and writes along c both coalesced.  F16: fp16 parts,
// hi = fp16(x), lo = fp16(x - hi); a value at or past fp16's range sets the
// status word.
template <bool F16>
__global__ void __launch_bounds__(256) transpose_split_kernel(const float *__restrict__ x,
                                                               float *__restrict__ hi,
                                                               float *__restrict__ lo, int C,
                                                               int T, int *status) {
  __shared__ float tile[32][33];
  const int t0 = blockIdx.x * 32, c0 = blockIdx.y * 32, b = blockIdx.z;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of 32
  const float *xb = x + (size_t)b * C * T;
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int t = t0 + tx;
    tile[r][tx] = (t < T && c0 + r < C) ? __ldcs(xb + (size_t)(c0 + r) * T + t) : 0.0f;
  }
  __syncthreads();
  const size_t ob = (size_t)b * T * C;
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int t = t0 + r;
    if (t < T && c0 + tx < C) {
      const float v = tile[tx][r];
      const size_t idx = ob + (size_t)t * C + c0 + tx;
      if constexpr (F16) {
        const __half h = __float2half_rn(v);
        reinterpret_cast<__half *>(hi)[idx] = h;
        reinterpret_cast<__half *>(lo)[idx] = __float2half_rn(v - __half2float(h));
        if (fabsf(v) >= 65504.0f && status) atomicExch(status, kStatusF16Range);
      } else {
        const float h = tf32_hi(v);
        hi[idx] = h;
        lo[idx] = v - h;
      }
    }
  }
}

}  // namespace

bv_status launch_transpose_split(const float *x, float *hi, float *lo, int B, int C, int T,
                                 cudaStream_t st, bool f16) {
  if (B <= 0 || T <= 0) return BV_OK;
  dim3 grid((T + 31) / 32, (C + 31) / 32, B);
  if (grid.y > 65535 || grid.z > 65535) return fail(BV_ERR_SHAPE, "transpose_split: grid");
  {
    LaunchTimer tm(st, "transpose_split", 0.0, (f16 ? 8.0 : 12.0) * B * C * T);
    if (f16)
      transpose_split_kernel<true><<<grid, 256, 0, st>>>(x, hi, lo, C, T, device_status_ptr());
    else
      transpose_split_kernel<false><<<grid, 256, 0, st>>>(x, hi, lo, C, T, nullptr);
  }
  count_launch();
  return check_launch("transpose_split_kernel");
}

bv_status launch_split_weights(const SplitTable &tab, cudaStream_t st) {
  if (tab.n <= 0) return BV_OK;
  if (tab.n > kMaxSplit) return fail(BV_ERR_SHAPE, "split_weights: %d entries", tab.n);
  double bytes = 0;
  for (int e = 0; e < tab.n; ++e) bytes += 12.0 * tab.count[e];
  {
    LaunchTimer tm(st, "weight_split", 0.0, bytes);
    split_weights_kernel<<<dim3(64, tab.n), 256, 0, st>>>(tab, device_status_ptr());
  }
  count_launch();
  return check_launch("split_weights_kernel");
}

bv_status launch_conv1d_tc(const float *x, int B, int Cin, int T, const float *w,
                           const float *w_split, const float *bias, int Cout, int K, int dil,
                           int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                           cudaStream_t st) {
  const double outs = (double)B * Cout * y_len;
  const OutMap om{1, 0, y_len, 1};
  return launch_tc_impl("conv1d_tc", x, B, Cin, T, w_split ? w_split : w, w_split != nullptr, Cout, bias, Cout, K, dil, pad, ep, y,
                        y_len, y_pitch, om, 2.0 * outs * Cin * K,
                        4.0 * ((double)B * Cin * T + (double)Cout * Cin * K +
                               outs * (1 + (ep.residual ? 1 : 0) + ep.accumulate)),
                        st);
}

int convt_taps(int K, int S) { return (K + S - 1) / S; }

bool conv_transpose1d_tc_supported(int Cin, int Cout, int K, int S) {
  const int nt = convt_taps(K, S);
  return conv1d_tc_supported(Cin, Cout, nt, 1);
}

size_t conv_transpose1d_tc_workspace(int Cin, int Cout, int K, int S) {
  return 2 * (size_t)S * Cout * Cin * convt_taps(K, S) * sizeof(float);  // wp and its lo part
}

bv_status launch_convt_pack_tc(const float *w, int Cin, int Cout, int K, int S, float *wp,
                               cudaStream_t st) {
  const int nt = convt_taps(K, S);
  const long long total = (long long)S * Cout * Cin * nt;
  {
    LaunchTimer tm(st, "convt_repack", 0.0, 8.0 * (double)total);
    const long long blocks = (total + 255) / 256;
    convt_repack_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st>>>(
        w, wp, wp + total, Cin, Cout, K, S, nt);
  }
  count_launch();
  return check_launch("convt_repack_kernel");
}

bv_status launch_conv_transpose1d_tc_packed(const float *x, int B, int Cin, int T,
                                            const float *wp, const float *bias, int Cout, int K,
                                            int S, int pad, float *y, cudaStream_t st) {
  const int nt = convt_taps(K, S);
  const int Tout = (T - 1) * S + K - 2 * pad;
  // phase r: conv output P (input-grid index, P < T + nt - 1) lands on sample
  // S P + r - pad
  const OutMap om{S, -pad, Tout, S};
  const Epi plain{nullptr, 1.0f, 0, 0};
  return launch_tc_impl("conv_transpose1d_tc", x, B, Cin, T, wp, true, S * Cout, bias, Cout,
                        nt, 1, nt - 1, plain, y, T + nt - 1, Tout, om,
                        2.0 * B * Cin * (double)Cout * K * T,
                        4.0 * ((double)B * Cin * T + (double)Cin * Cout * K +
                               (double)B * Cout * Tout),
                        st);
}

bv_status launch_conv_transpose1d_tc(const float *x, int B, int Cin, int T, const float *w,
                                     const float *bias, int Cout, int K, int S, int pad, float *y,
                                     float *wp, cudaStream_t st) {
  BV_TRY(launch_convt_pack_tc(w, Cin, Cout, K, S, wp, st));
  return launch_conv_transpose1d_tc_packed(x, B, Cin, T, wp, bias, Cout, K, S, pad, y, st);
}


bool conv1d_tm_supported(int Cin, int Cout, int K, int dil) {
  // input rows of Cin floats must be 16-byte multiples (TMA strides); a
  // partial last channel block costs padded tensor work, so at most a third.
  // From 40 output channels, or 32 when neither the tile nor the channel
  // blocks are padded.  Measured on B200 against the FP32 narrow kernel: 24
  // channels in 32-channel tiles and blocks break even per conv and lose with
  // the dearer time-major activation (60 s H3 decode 565 -> 560 audio-s/s);
  // the 32-channel stage of the LTX bandwidth-extension tail gains (10.0 ->
  // 9.3 ms per 10 s).  A reduction of two channel blocks (a one-tap conv over
  // 64 channels) already beats the SIMT kernel (measured on the DAV decoder's
  // 96-channel one-tap convs).
  return Cin % 4 == 0 && 3 * tm_cin_pad(Cin) <= 4 * Cin &&
         (Cout >= 40 || (Cout == 32 && Cin % 32 == 0)) &&
         tm_cin_pad(Cin) * K >= 64 && K >= 1 && K <= MAX_K && dil >= 1 &&
         (K - 1) * dil <= TM_MAX_HALO && encode_fn() != nullptr;
}

namespace {

// The time-major launch: w_split holds hi then lo of a [w_rows, K Cp] tap-major
// matrix (w_rows = phases Cout), outputs go through om.
bv_status tm_impl(const char *cls, const float *x_hi, const float *x_lo, int B, int Cin, int T,
                  const float *w_split, int w_rows, const float *bias, int Cout, int K, int dil,
                  int pad, const Epi &ep, float *y, int y_len, int y_pitch, const OutMap &om,
                  double flops, double bytes, cudaStream_t st, bool f16 = false) {
  const int nt = pick_nt_pair(Cout);
  // tap-major weight row, padded channels
  const int KK = (f16 ? tm_cin_pad_f16(Cin) : tm_cin_pad(Cin)) * K;
  CUtensorMap xh, xl, wh, wl;
  BV_TRY(encode_x_tm(&xh, x_hi, B, Cin, T, BM + (K - 1) * dil, f16));
  BV_TRY(encode_x_tm(&xl, x_lo, B, Cin, T, BM + (K - 1) * dil, f16));
  // each CTA of a pair loads half the rows; lo follows hi
  const float *w_lo = reinterpret_cast<const float *>(reinterpret_cast<const char *>(w_split) +
                                                      (size_t)w_rows * KK * (f16 ? 2 : 4));
  BV_TRY(encode_w(&wh, w_split, w_rows, KK, nt / 2, f16));
  BV_TRY(encode_w(&wl, w_lo, w_rows, KK, nt / 2, f16));
  bv_status s;
  {
    LaunchTimer tm(st, cls, flops, bytes);
#define BV_TM_RUN(N, TP, H)                                                                 \
  run_tm<N, TP, H>(xh, xl, wh, wl, B, Cin, bias, Cout, K, dil, pad, ep, y, y_len, y_pitch, om, st)
#define BV_TM_CASE(N)                                                                       \
  case N:                                                                                   \
    s = f16 ? (K >= 3 ? BV_TM_RUN(N, 4, true) : BV_TM_RUN(N, 2, true))                      \
            : (K >= 3 ? BV_TM_RUN(N, 4, false) : BV_TM_RUN(N, 2, false));                   \
    break;
    switch (nt) {
      BV_TM_CASE(32)
      BV_TM_CASE(64)
      BV_TM_CASE(96)
      BV_TM_CASE(128)
      default:
        return fail(BV_ERR_UNSUPPORTED, "conv1d_tm: tile %d", nt);
    }
#undef BV_TM_CASE
#undef BV_TM_RUN
  }
  if (s != BV_OK) return s;
  count_launch();
  return check_launch("conv1d_tm_kernel");
}

}  // namespace

bool tm_f16_ok(int Cin) {
  return Cin % 8 == 0 && 3 * tm_cin_pad_f16(Cin) <= 4 * Cin && activation_tm_supported(Cin);
}

bv_status launch_conv1d_tm(const float *x_hi, const float *x_lo, int B, int Cin, int T,
                           const float *w_split, const float *bias, int Cout, int K, int dil,
                           int pad, const Epi &ep, float *y, int y_len, int y_pitch,
                           cudaStream_t st, bool f16) {
  if (B <= 0 || y_len <= 0) return BV_OK;
  if (!conv1d_tm_supported(Cin, Cout, K, dil) || (f16 && !tm_f16_ok(Cin)))
    return fail(BV_ERR_UNSUPPORTED, "conv1d_tm: Cin %d Cout %d K %d%s", Cin, Cout, K,
                f16 ? " (fp16)" : "");
  // algorithmic work: the useful products (Cin K per output), not the padded
  // channel block or the three 3xTF32 terms
  const double outs = (double)B * Cout * y_len;
  return tm_impl(f16 ? "conv1d_tm_f16" : "conv1d_tm", x_hi, x_lo, B, Cin, T, w_split, Cout, bias,
                 Cout, K, dil, pad, ep,
                 y, y_len, y_pitch, OutMap{1, 0, y_len, 1}, 2.0 * outs * Cin * K,
                 4.0 * ((double)B * Cin * T + (double)Cout * Cin * K +
                        outs * (1 + (ep.residual ? 1 : 0) + ep.accumulate)),
                 st, f16);
}

bool conv_transpose1d_tm_supported(int Cin, int Cout, int K, int S) {
  return conv1d_tm_supported(Cin, Cout, convt_taps(K, S), 1);
}

size_t conv_transpose1d_tm_workspace(int Cin, int Cout, int K, int S) {
  return 2 * (size_t)S * Cout * tm_cin_pad(Cin) * convt_taps(K, S) * sizeof(float);
}

bv_status launch_convt_pack_tm(const float *w, int Cin, int Cout, int K, int S, float *wp,
                               cudaStream_t st, bool f16) {
  const int nt = convt_taps(K, S), cp = f16 ? tm_cin_pad_f16(Cin) : tm_cin_pad(Cin);
  const long long total = (long long)S * Cout * nt * cp;
  // lo follows hi: total values of 4 (tf32) or 2 (fp16) bytes
  float *wp_lo = reinterpret_cast<float *>(reinterpret_cast<char *>(wp) + total * (f16 ? 2 : 4));
  {
    LaunchTimer tm(st, "convt_repack", 0.0,
                   4.0 * (double)Cin * Cout * K + (f16 ? 4.0 : 8.0) * (double)total);
    const long long blocks = (total + 255) / 256;
    convt_repack_tm_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, st>>>(
        w, wp, wp_lo, Cin, Cout, K, S, nt, cp, f16 ? 1 : 0, device_status_ptr());
  }
  count_launch();
  return check_launch("convt_repack_tm_kernel");
}

bv_status launch_conv_transpose1d_tm_packed(const float *x_hi, const float *x_lo, int B, int Cin,
                                            int T, const float *wp, const float *bias, int Cout,
                                            int K, int S, int pad, float *y, cudaStream_t st,
                                            bool f16) {
  if (B <= 0 || T <= 0) return BV_OK;
  if (!conv_transpose1d_tm_supported(Cin, Cout, K, S) || (f16 && !tm_f16_ok(Cin)))
    return fail(BV_ERR_UNSUPPORTED, "conv_transpose1d_tm: Cin %d Cout %d%s", Cin, Cout,
                f16 ? " (fp16)" : "");
  const int nt = convt_taps(K, S);
  const int Tout = (T - 1) * S + K - 2 * pad;
  // phase r: conv output P (input-grid index, P < T + nt - 1) lands on sample
  // S P + r - pad of the output row
  return tm_impl(f16 ? "conv_transpose1d_tm_f16" : "conv_transpose1d_tm", x_hi, x_lo, B, Cin, T,
                 wp, S * Cout, bias, Cout, nt, 1, nt - 1, Epi{nullptr, 1.0f, 0, 0}, y, T + nt - 1,
                 Tout, OutMap{S, -pad, Tout, S}, 2.0 * B * Cin * (double)Cout * K * T,
                 4.0 * ((double)B * Cin * T + (double)Cin * Cout * K + (double)B * Cout * Tout),
                 st, f16);
}

bv_status launch_conv_transpose1d_tm(const float *x_hi, const float *x_lo, int B, int Cin, int T,
                                     const float *w, const float *bias, int Cout, int K, int S,
                                     int pad, float *y, float *wp, cudaStream_t st, bool f16) {
  if (B <= 0 || T <= 0) return BV_OK;
  if (!conv_transpose1d_tm_supported(Cin, Cout, K, S) || (f16 && !tm_f16_ok(Cin)))
    return fail(BV_ERR_UNSUPPORTED, "conv_transpose1d_tm: Cin %d Cout %d", Cin, Cout);
  BV_TRY(launch_convt_pack_tm(w, Cin, Cout, K, S, wp, st, f16));
  return launch_conv_transpose1d_tm_packed(x_hi, x_lo, B, Cin, T, wp, bias, Cout, K, S, pad, y,
                                           st, f16);
}

}  // namespace bv
