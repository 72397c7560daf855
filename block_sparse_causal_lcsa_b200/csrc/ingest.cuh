// Block-granular pass over a chunk's token tensors: mean-pooling (FlashVSR
// summary, section 2.2 stage 2: average pooling of 2x8x8 blocks gives the
// compact block features of the coarse map) fused with the streaming KV-cache
// write (section 2.2 stage 3: later layers keep a KV cache; section 3: the
// stream advances 2 latent frames at a time).
//
// One CTA of 256 threads owns one 2x8x8 block of one tensor and, per its
// role, pools it (a float64 row of D means), copies it into the ring cache,
// or both. K is read once for both its pooled row and its cache copy, so a
// streaming step reads each of Q, K, V from HBM exactly once. A block is 16
// runs of 8 tokens x D bf16 (2 KB for D = 128) in the [T][Y][X][D] layout:
// each warp-wide 16-byte load covers whole contiguous token rows, every load
// of the CTA is issued before the first add or store (D/16 x 16 bytes in flight
// per thread), lanes accumulate 8 channels in float64, lanes of the same
// channels are combined with shuffles and the 8 warps in shared memory. The sum
// of at most 128 bf16 values is exact in float64 (when the block's non-zero
// values span at most 38 binades), so the mean does not depend on the order of
// accumulation.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

struct IngestTensor {
  const __nv_bfloat16* src;   // [B][H][T][Y][X][D], D unit stride
  int64_t sb, sh, st, sy, sx;
  int32_t T, nT;              // frames, temporal blocks ceil(T/2) (oldest has one frame if T is odd)
  int32_t tb_first;           // blocks [tb_first, nT) are processed
  int64_t units;              // B * H * (nT - tb_first) * Hb * Wb
  double* pool_out;           // NULL: no pooling
  int32_t pool_ring;          // 0: pool_out is [B][H][nT][Hb][Wb][D]; 1: the cache's pooled ring
  __nv_bfloat16* copy_dst;    // NULL: no copy; else the cache ring [B][H][cap][Y][X][D]
};

struct IngestParams {
  IngestTensor t[3];
  int32_t H, Y, X, Hb, Wb;
  int32_t cap, stream_offset;   // ring capacity (frames) and first cache stream
  int64_t first_abs[64];        // absolute frame of chunk frame 0, per chunk stream
};

constexpr int INGEST_THREADS = 256;
constexpr int INGEST_WARPS = INGEST_THREADS / 32;

template <int D>
__global__ void __launch_bounds__(INGEST_THREADS)
ingest_kernel(const __grid_constant__ IngestParams p) {
  constexpr int VPT = D / 8;                                    // 16-byte vectors per token
  constexpr int NV = 128 * VPT / INGEST_THREADS;                // vectors per thread
  static_assert(NV * INGEST_THREADS == 128 * VPT, "block must split evenly");
  __shared__ double part[INGEST_WARPS][D];

  // 32-bit index arithmetic (the grid is below 2^31 blocks): every thread
  // derives its block before it can issue a load
  int unit = static_cast<int>(blockIdx.x);
  int which = 0;
  while (which < 2 && unit >= p.t[which].units) {
    unit -= static_cast<int>(p.t[which].units);
    ++which;
  }
  const IngestTensor& tt = p.t[which];
  const int HbWb = p.Hb * p.Wb;
  const int nb = tt.nT - tt.tb_first;
  const int sp = unit % HbWb;
  int rest = unit / HbWb;
  const int tb = tt.tb_first + rest % nb;
  rest /= nb;
  const int h = rest % p.H;
  const int bn = rest / p.H;
  const int yb = sp / p.Wb, xb = sp % p.Wb;
  const int f0 = tt.T - 2 * tt.nT + 2 * tb;                     // older frame (-1: missing)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int vec = tid % VPT;                                    // fixed channel group of this thread

  const __nv_bfloat16* base = tt.src + bn * tt.sb + h * tt.sh +
                              static_cast<int64_t>(8 * yb) * tt.sy +
                              static_cast<int64_t>(8 * xb) * tt.sx + vec * 8;
  uint4 raw[NV];
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int tok = (u * INGEST_THREADS + tid) / VPT;
    const int f = f0 + (tok >> 6);
    raw[u] = f >= 0 ? __ldg(reinterpret_cast<const uint4*>(
                          base + static_cast<int64_t>(f) * tt.st + ((tok >> 3) & 7) * tt.sy +
                          (tok & 7) * tt.sx))
                    : make_uint4(0u, 0u, 0u, 0u);
  }

  if (tt.copy_dst != nullptr) {
    const int64_t cb = bn + p.stream_offset;
    // ring slots of the block's two frames, once per thread (the host passes
    // first_abs in [0, cap), so the frame numbers fit in 32 bits)
    const int abs0 = static_cast<int>(p.first_abs[bn]);
    const int slot_old = f0 >= 0 ? (abs0 + f0) % p.cap : 0;
    const int slot_new = (abs0 + f0 + 1) % p.cap;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const int tok = (u * INGEST_THREADS + tid) / VPT;
      const int f = f0 + (tok >> 6);
      if (f < 0) continue;
      const int64_t slot = (tok >> 6) ? slot_new : slot_old;
      const int64_t row = ((cb * p.H + h) * p.cap + slot) * p.Y + 8 * yb + ((tok >> 3) & 7);
      *reinterpret_cast<uint4*>(tt.copy_dst + (row * p.X + 8 * xb + (tok & 7)) * D + vec * 8) = raw[u];
    }
  }

  if (tt.pool_out != nullptr) {
    double acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f2 = __bfloat1622float2(v2[k]);
        acc[2 * k] += static_cast<double>(f2.x);
        acc[2 * k + 1] += static_cast<double>(f2.y);
      }
    }
#pragma unroll
    for (int m = VPT; m < 32; m <<= 1) {
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], m);
    }
    if (lane < VPT) {
#pragma unroll
      for (int k = 0; k < 8; ++k) part[warp][vec * 8 + k] = acc[k];
    }
    __syncthreads();
    if (tid < D) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < INGEST_WARPS; ++w) s += part[w][tid];
      const double inv = f0 < 0 ? (1.0 / 64.0) : (1.0 / 128.0);  // exact powers of two
      int64_t row;
      if (tt.pool_ring) {
        // the chunk ends at absolute frame first_abs + T (even): its block tb
        // is absolute block (first_abs + T)/2 - nT + tb
        const int64_t m = (p.first_abs[bn] + tt.T) / 2 - tt.nT + tb;
        row = ((static_cast<int64_t>(bn) + p.stream_offset) * p.H + h) * (p.cap / 2) + m % (p.cap / 2);
      } else {
        row = (static_cast<int64_t>(bn) * p.H + h) * tt.nT + tb;
      }
      tt.pool_out[(row * HbWb + sp) * D + tid] = s * inv;
    }
  }
}

}  // namespace lcsa
