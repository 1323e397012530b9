// Tile gather / stitch launchers for the tiled decode.
#pragma once

#include "common.cuh"

namespace bv {

// Decoded tiles, in up to two groups of equal-length tiles.
struct TileGroups {
  int n;                      // groups in use (1 or 2)
  const float *data[2];       // [count * B, O, pitch], rows (k - k0) B + b
  long long k0[2];            // first tile index of the group
  long long count[2];         // tiles in the group
  long long len_samples[2];   // tile length in samples
  long long pitch[2];         // row pitch in samples (>= len_samples)
  long long max_len_samples;  // longest tile
};

// zt[u - u0, c, f] = z[b, c, k step + f] for units u = k B + b in [u0, u0 + n_units), tiles of
// `len` frames.
bv_status launch_gather_tiles(const float *z, float *zt, int B, int C, int frames, int step,
                              int len, long long u0, long long n_units, cudaStream_t st);

bv_status launch_stitch_tiles(const TileGroups &g, float *y, int B, int O, long long L,
                              int step_samples, cudaStream_t st);

}  // namespace bv
