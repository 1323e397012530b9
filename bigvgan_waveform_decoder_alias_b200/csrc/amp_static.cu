// bv_amp_block_static: the AMP block for callers that cannot allocate.
//
// Some callers have no way to hand the library a workspace.  An audio
// plugin's render callback or any real-time thread must not call cudaMalloc:
// it can block while the driver takes locks or synchronises the device, and a
// missed deadline is an audible dropout.  Hosts that fix their device memory
// budget up front, or that run the decoder while another component owns the
// allocator, are in the same position.  This entry point keeps its scratch in
// a file-scope device array compiled into the library, so the caller passes
// only its inputs and outputs.
//
// The array is BV_AMP_STATIC_MAX_ELEMS floats per scratch tensor, three
// tensors (12 MiB), and every GPU that loads the library holds it until the
// process exits.  Host code cannot use the array's name as a device address;
// the first call on each device resolves the address with
// cudaGetSymbolAddress while that device is current, and later calls reuse it.
#include <mutex>

#include "bv.h"
#include "common.cuh"

namespace {

constexpr size_t kScratchFloats = 3 * (size_t)BV_AMP_STATIC_MAX_ELEMS;

// Scratch for the three intermediate tensors of one AMP block.  Shared by all
// calls; every element a call reads was written earlier in the same call, so
// nothing needs clearing between calls.
static __device__ __align__(256) float g_amp_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_amp_scratch on the current device, resolved once.
bv_status scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return bv::fail(BV_ERR_CUDA, "bv_amp_block_static: no CUDA device: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return bv::fail(BV_ERR_UNSUPPORTED, "bv_amp_block_static: device %d beyond %d", dev,
                    kMaxDevices);
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_amp_scratch);
    if (e != cudaSuccess || !p)
      return bv::fail(BV_ERR_CUDA, "bv_amp_block_static: cudaGetSymbolAddress: %s",
                      cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return BV_OK;
}

}  // namespace

extern "C" bv_status bv_amp_block_static(const float *x, int B, int C, int T,
                                         const bv_amp_params *p, float *y, float scale,
                                         int accumulate, void *stream) {
  if (B < 1 || C < 1 || T < 1)
    return bv::fail(BV_ERR_SHAPE, "bv_amp_block_static: B=%d C=%d T=%d", B, C, T);
  const unsigned long long n = (unsigned long long)B * C * T;
  if (n > (unsigned long long)BV_AMP_STATIC_MAX_ELEMS)
    return bv::fail(BV_ERR_WORKSPACE,
                    "bv_amp_block_static: B*C*T = %llu exceeds the static scratch limit of %d "
                    "elements; use bv_amp_block with a workspace",
                    n, BV_AMP_STATIC_MAX_ELEMS);
  void *scratch = nullptr;
  const bv_status st = scratch_address(&scratch);
  if (st != BV_OK) return st;
  return bv_amp_block(x, B, C, T, p, y, scale, accumulate, scratch,
                      kScratchFloats * sizeof(float), stream);
}
