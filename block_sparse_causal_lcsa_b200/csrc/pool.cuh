// Block mean-pooling of Q and K over 2x8x8 (t, y, x) token blocks
// (FlashVSR summary, section 2.2 stage 2: average pooling gives compact
// block-level features for the coarse block map).
//
// HBM-bound: every input byte is read once with 16-byte coalesced loads and
// each block writes D float64 means. One CTA of 4 warps owns one block; each
// warp takes 32 of its 128 tokens and issues all of its loads before the first
// add (16 x 16 bytes in flight per lane for D = 128), so one block costs about
// one memory round trip. Lanes accumulate 8 channels in float64, the warp's
// token halves are combined with shuffles and the 4 warps' partial sums are
// added in shared memory. The sum of at most 128 bf16 values is exact in
// float64 (when the block's non-zero values span at most 38 binades), so the
// result does not depend on the order of accumulation and equals the
// correctly rounded mean.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

struct PoolTensor {
  const __nv_bfloat16* data;
  double* out;          // [B][H][nT][Hb][Wb][D]
  int64_t sb, sh, st, sy, sx;
  int32_t T;            // frames
  int32_t nT;           // temporal blocks = ceil(T/2)
  int64_t units;        // B*H*nT*Hb*Wb
};

struct PoolParams {
  PoolTensor t[2];      // Q, then K (units of K may be 0)
  int32_t H, Hb, Wb;
};

constexpr int POOL_WARPS = 4;
constexpr int POOL_THREADS = POOL_WARPS * 32;

template <int D>
__global__ void __launch_bounds__(POOL_THREADS)
pool_kernel(const __grid_constant__ PoolParams p) {
  constexpr int LANES_PER_TOKEN = D / 8;            // 16 B (8 bf16) per lane
  constexpr int TOKENS_PER_STEP = 32 / LANES_PER_TOKEN;
  constexpr int TOKENS_PER_WARP = 128 / POOL_WARPS;
  constexpr int STEPS = TOKENS_PER_WARP / TOKENS_PER_STEP;
  __shared__ double part[POOL_WARPS][D];

  const int64_t unit_all = blockIdx.x;
  const int which = unit_all < p.t[0].units ? 0 : 1;
  const int64_t unit = which == 0 ? unit_all : unit_all - p.t[0].units;
  const PoolTensor& tt = p.t[which];

  const int HbWb = p.Hb * p.Wb;
  const int sp = static_cast<int>(unit % HbWb);
  const int64_t rest = unit / HbWb;
  const int tb = static_cast<int>(rest % tt.nT);
  const int64_t bh = rest / tt.nT;
  const int64_t b = bh / p.H, h = bh % p.H;
  const int yb = sp / p.Wb, xb = sp % p.Wb;
  const int f0 = tt.T - 2 * tt.nT + 2 * tb;         // older frame of the block (-1: missing)
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int chan = (lane % LANES_PER_TOKEN) * 8;
  const int sub = lane / LANES_PER_TOKEN;

  const __nv_bfloat16* base = tt.data + b * tt.sb + h * tt.sh +
                              static_cast<int64_t>(8 * yb) * tt.sy +
                              static_cast<int64_t>(8 * xb) * tt.sx + chan;
  double acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0;

  // Tokens are numbered (frame, y, x); warp w owns tokens [32w, 32w+32).
  // With a missing older frame the first 64 tokens do not exist.
  const bool active = !(f0 < 0 && warp < POOL_WARPS / 2);
  if (active) {
    uint4 raw[STEPS];
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      const int tok = warp * TOKENS_PER_WARP + s * TOKENS_PER_STEP + sub;
      const int f = f0 + (tok >> 6);
      const int yy = (tok >> 3) & 7, xx = tok & 7;
      raw[s] = __ldg(reinterpret_cast<const uint4*>(
          base + static_cast<int64_t>(f) * tt.st + yy * tt.sy + xx * tt.sx));
    }
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&raw[s]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f2 = __bfloat1622float2(v2[k]);
        acc[2 * k] += static_cast<double>(f2.x);
        acc[2 * k + 1] += static_cast<double>(f2.y);
      }
    }
  }
#pragma unroll
  for (int m = LANES_PER_TOKEN; m < 32; m <<= 1) {
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], m);
  }
  if (sub == 0) {
#pragma unroll
    for (int k = 0; k < 8; ++k) part[warp][chan + k] = acc[k];
  }
  __syncthreads();
  const double inv = (f0 < 0) ? (1.0 / 64.0) : (1.0 / 128.0);  // exact powers of two
  for (int c = threadIdx.x; c < D; c += POOL_THREADS) {
    double s = 0.0;
#pragma unroll
    for (int w = 0; w < POOL_WARPS; ++w) s += part[w][c];
    tt.out[unit * D + c] = s * inv;
  }
}

}  // namespace lcsa
