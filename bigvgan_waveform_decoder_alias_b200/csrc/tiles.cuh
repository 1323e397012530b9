// Tile gather / stitch launchers for the tiled decode.
#pragma once

#include "common.cuh"

namespace bv {

// Decoded tiles, in up to two groups of equal-length tiles.
struct TileGroups {
  int n;                      // groups in use (1 or 2)
  const float *data[2];       // [count * B, O, len_samples]
  long long k0[2];            // first tile index of the group
  long long count[2];         // tiles in the group
  long long len_samples[2];   // tile length in samples
  long long max_len_samples;  // longest tile
};

bv_status launch_gather_tiles(const float *z, float *zt, int B, int C, int frames, int step,
                              int len, int k0, int n_tiles, cudaStream_t st);

bv_status launch_stitch_tiles(const TileGroups &g, float *y, int B, int O, long long L,
                              int step_samples, cudaStream_t st);

}  // namespace bv
