// Block lists for dense attention confined to one segment (FlashVSR summary,
// section 2.2 stage 1: joint video-image training with a block-diagonal
// segment mask, so that attention stays inside one video clip or one image;
// an image is a one-frame video).
//
// A segment is one stream of the cache: its frames [begin, end). Segments of
// different lengths share one query tensor of Tq frames: segment b's frames
// are the newest end-begin of them, older query frames are padding. Every
// query block that holds at least one of the segment's frames keeps every key
// block of the segment (no causal limit, no top-K), in ascending order; a
// query block of padding only keeps none. The lists feed the same attention
// kernels (forward and backward) as the sparse path.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

struct SegmentParams {
  int32_t* blk_idx;     // [B*H][nQB][kmax]
  int32_t* blk_cnt;     // [B*H][nQB]
  int32_t H, Tq, nQT, HbWb, kmax;
  int64_t rows;         // B*H*nQB
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

// One warp per query block row.
__global__ void __launch_bounds__(256) segment_blocks_kernel(const __grid_constant__ SegmentParams p) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nQB = p.nQT * p.HbWb;
  if (row >= p.rows) return;
  const int bh = static_cast<int>(row / nQB);
  const int qb = static_cast<int>(row % nQB);
  const int b = bh / p.H;
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  const int64_t frames = end - begin;
  const int tq = qb / p.HbWb;
  const int f_newer = p.Tq - 2 * p.nQT + 2 * tq + 1;       // newer frame of the query block
  const bool real = f_newer >= p.Tq - frames;               // it belongs to the segment
  const int nkb = real ? static_cast<int>((end >> 1) - (begin >> 1)) * p.HbWb : 0;
  int32_t* out = p.blk_idx + row * p.kmax;
  for (int j = lane; j < p.kmax; j += 32) out[j] = j < nkb ? j : -1;
  if (lane == 0) p.blk_cnt[row] = nkb;
}

}  // namespace lcsa
