// Token reordering: gather or scatter whole rows of [n_mats, L, row] tensors
// by an index vector, and the 3-D Hilbert-curve order that feeds it.
//
// The SpargeAttn article ("Hilbert 曲线置换" under its technical details)
// reorders the T x H x W tokens of a video along a 3-D Hilbert curve before
// attention, so that a tile of consecutive tokens is a compact 3-D region and
// more tiles can be skipped.  Attention without a causal mask commutes with a
// common reordering of Q, K and V, so O and lse come back to the original
// order by the inverse (scatter) of the same permutation.
//
// The copy is pure HBM traffic: 16-byte vector loads and stores, consecutive
// threads on consecutive 16-byte chunks of one row, so both the gathered reads
// (one row is 128 or 256 contiguous bytes) and the writes are coalesced; a
// grid-stride loop over all chunks sized to the SM count.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace sskip {

template <typename Chunk>
__global__ void __launch_bounds__(256)
    permute_rows_kernel(const Chunk* __restrict__ src, Chunk* __restrict__ dst,
                        const int32_t* __restrict__ idx, long long n_mats, int L,
                        int chunks_per_row, int scatter) {
  const long long per_mat = (long long)L * chunks_per_row;
  const long long total = n_mats * per_mat;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total;
       c += (long long)gridDim.x * blockDim.x) {
    const long long m = c / per_mat;
    const long long rem = c - m * per_mat;
    const int i = (int)(rem / chunks_per_row);
    const int e = (int)(rem - (long long)i * chunks_per_row);
    const int j = __ldg(idx + i);
    if (j < 0 || j >= L) {  // not a permutation of 0 .. L-1: record it, touch nothing
      latch_status(kStatusInvalidArg);
      continue;
    }
    const long long a = (m * L + i) * chunks_per_row + e;   // position i
    const long long b = (m * L + j) * chunks_per_row + e;   // position idx[i]
    if (scatter) dst[b] = src[a];
    else dst[a] = src[b];
  }
}

}  // namespace sskip
