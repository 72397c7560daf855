// Streaming KV-cache append (FlashVSR summary, section 2.2 stage 3: later
// layers refine temporal consistency through a KV cache; section 3: the
// stream advances in chunks of 8 video frames = 2 latent frames).
//
// The cache is a ring of frames per (stream, head): absolute frame a lives in
// slot a % cap_frames and the pooled K of block m (frames 2m, 2m+1) in slot
// m % (cap_frames/2). Appending writes the chunk's frames into their slots
// (overwriting evicted ones) and copies the chunk's pooled K blocks; the host
// advances begin/end. HBM-bound copy organised by planes: a K or V plane is
// one (stream, head, frame) = Y*X*D contiguous bf16 in the cache, a pooled
// plane one (stream, head, block row of a frame pair) = Hb*Wb*D doubles.
// grid.y enumerates planes, grid.x chunks of 16-byte vectors within a plane,
// so address decoding happens once per CTA and the copy loop is plain
// 16-byte loads and stores (8 in flight per thread).
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

struct AppendParams {
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const double* kp_new;                 // [Bn][H][nTn][Hb][Wb][D]
  __nv_bfloat16* k_cache;               // [B][H][cap][Y][X][D]
  __nv_bfloat16* v_cache;
  double* kp_cache;                     // [B][H][cap/2][Hb][Wb][D]
  int64_t ksb, ksh, kst, ksy, ksx;      // strides of k_new (elements)
  int64_t vsb, vsh, vst, vsy, vsx;      // strides of v_new
  int32_t Bn, H, Y, X, D, Hb, Wb;
  int32_t cap, stream_offset;
  int32_t f_first, n_frames;            // chunk frames [f_first, f_first+n_frames) are copied
  int32_t nTn, tb_first;                // chunk blocks [tb_first, nTn) are copied
  int32_t kv_planes, pool_planes;       // Bn*H*n_frames, Bn*H*(nTn-tb_first)
  int64_t first_abs[64];                // absolute frame of chunk frame 0, per stream bn
};

constexpr int APPEND_THREADS = 256;
constexpr int APPEND_VPT = 8;           // 16-byte vectors per thread per CTA
constexpr int APPEND_CHUNK = APPEND_THREADS * APPEND_VPT;

__global__ void __launch_bounds__(APPEND_THREADS)
kv_append_kernel(const __grid_constant__ AppendParams p) {
  const int plane = blockIdx.y;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * APPEND_CHUNK;
  if (plane < 2 * p.kv_planes) {
    const bool is_v = plane >= p.kv_planes;
    int r = is_v ? plane - p.kv_planes : plane;
    const int f = p.f_first + r % p.n_frames; r /= p.n_frames;
    const int h = r % p.H;
    const int bn = r / p.H;
    const int64_t b = bn + p.stream_offset;
    const int64_t slot = (p.first_abs[bn] + f) % p.cap;
    const int vpr = p.D / 8;                                 // vectors per token row
    const int64_t plane_vecs = static_cast<int64_t>(p.Y) * p.X * vpr;
    if (v0 >= plane_vecs) return;
    const int64_t sb = is_v ? p.vsb : p.ksb, sh = is_v ? p.vsh : p.ksh;
    const int64_t st = is_v ? p.vst : p.kst, sy = is_v ? p.vsy : p.ksy;
    const int64_t sx = is_v ? p.vsx : p.ksx;
    const __nv_bfloat16* src = (is_v ? p.v_new : p.k_new) + bn * sb + h * sh + f * st;
    uint4* dst = reinterpret_cast<uint4*>((is_v ? p.v_cache : p.k_cache) +
                                          ((b * p.H + h) * p.cap + slot) * plane_vecs * 8);
    const bool flat = (sx == p.D) && (sy == static_cast<int64_t>(p.X) * p.D);
    uint4 buf[APPEND_VPT];
#pragma unroll
    for (int u = 0; u < APPEND_VPT; ++u) {
      const int64_t v = v0 + u * APPEND_THREADS + threadIdx.x;
      if (v < plane_vecs) {
        int64_t off;
        if (flat) {
          off = v * 8;
        } else {
          const int row = static_cast<int>(v / vpr), vec = static_cast<int>(v % vpr);
          off = static_cast<int64_t>(row / p.X) * sy + static_cast<int64_t>(row % p.X) * sx +
                vec * 8;
        }
        buf[u] = __ldg(reinterpret_cast<const uint4*>(src + off));
      }
    }
#pragma unroll
    for (int u = 0; u < APPEND_VPT; ++u) {
      const int64_t v = v0 + u * APPEND_THREADS + threadIdx.x;
      if (v < plane_vecs) dst[v] = buf[u];
    }
  } else {
    int r = plane - 2 * p.kv_planes;
    const int nt = p.nTn - p.tb_first;
    const int tb = p.tb_first + r % nt; r /= nt;
    const int h = r % p.H;
    const int bn = r / p.H;
    const int64_t b = bn + p.stream_offset;
    // The chunk ends at absolute frame first_abs + f_first + n_frames (even),
    // so its block tb is absolute block end/2 - nTn + tb.
    const int64_t end_abs = p.first_abs[bn] + p.f_first + p.n_frames;
    const int64_t m = end_abs / 2 - p.nTn + tb;
    const int64_t slot = m % (p.cap / 2);
    const int64_t plane_vecs = static_cast<int64_t>(p.Hb) * p.Wb * p.D / 2;  // 16-byte vectors
    const uint4* src = reinterpret_cast<const uint4*>(
        p.kp_new + ((static_cast<int64_t>(bn) * p.H + h) * p.nTn + tb) * plane_vecs * 2);
    uint4* dst = reinterpret_cast<uint4*>(
        p.kp_cache + ((b * p.H + h) * (p.cap / 2) + slot) * plane_vecs * 2);
#pragma unroll
    for (int u = 0; u < APPEND_VPT; ++u) {
      const int64_t v = v0 + u * APPEND_THREADS + threadIdx.x;
      if (v < plane_vecs) dst[v] = __ldg(src + v);
    }
  }
}

}  // namespace lcsa
