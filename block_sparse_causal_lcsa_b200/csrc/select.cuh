// Coarse block map, causal and locality masks, and top-K selection
// (FlashVSR summary, section 2.2 stage 2: coarse block-to-block attention map,
// keep the top-K block pairs, causal masking; section 2.3: a spatial window
// per query with a boundary-truncate or boundary-preserve rule).
//
// One CTA (4 warps) owns SEL_ROWS query blocks of one (stream, head, temporal
// block) and all of their causal candidates.
// Phase 1: each thread takes candidates in turn, streams the candidate's
//   pooled key row from L2 and scores it against all SEL_ROWS query rows held
//   in shared memory: SEL_ROWS independent float64 chains, each summed in
//   channel order with every product rounded before it is added (no fused
//   multiply-add), then divided by sqrt(D) - the same float64 value as the
//   definition, bit for bit. Scores become order-preserving 64-bit keys;
//   blocks outside the window get key 0, below every finite score.
// Phase 2: one warp per query block finds the K-th largest key exactly with an
//   8-pass, 8-bit radix select (256-bin shared-memory histogram per pass,
//   warp suffix scan), then one ascending pass keeps every block above
//   tau+eps and the lowest-index blocks of the band [tau-eps, tau+eps].
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int SEL_ROWS = 4;       // query blocks per CTA (one warp each in phase 2)
constexpr int SEL_THREADS = SEL_ROWS * 32;

struct SelectParams {
  const double* q_pool;   // [B][H][nQT][Hb][Wb][D]
  const double* k_pool;   // ring [B][H][cap_blk][Hb][Wb][D]
  int32_t* blk_idx;       // [B][H][nQT*Hb*Wb][kmax]
  int32_t* blk_cnt;       // [B][H][nQT*Hb*Wb]
  int32_t H, Hb, Wb, nQT, cap_blk;
  int32_t top_k, window, window_mode, kmax;
  int32_t c_stride;       // row stride (keys) of the key buffer in shared memory
  double density, tie_eps, sqrt_d;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

__host__ __device__ constexpr size_t select_smem_bytes(int D, int c_stride) {
  return sizeof(double) * SEL_ROWS * D + sizeof(uint32_t) * SEL_ROWS * 256 +
         sizeof(uint64_t) * static_cast<size_t>(SEL_ROWS) * c_stride;
}

__device__ __forceinline__ uint64_t order_key(double s) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(s));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
  const uint64_t u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double(static_cast<long long>(u));
}

__device__ __forceinline__ void window_bounds(int i, int n, int w, int mode, int& lo, int& hi) {
  if (w <= 0) { lo = 0; hi = n; return; }
  const int r = w / 2;
  if (mode == 0) {  // truncate at the frame edge
    lo = max(0, i - r);
    hi = min(n, i + r + 1);
  } else {          // preserve: shift inward, keep w blocks
    lo = max(0, min(i - r, n - w));
    hi = min(n, lo + w);
  }
}

template <int D>
__global__ void __launch_bounds__(SEL_THREADS)
select_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  double* qs = reinterpret_cast<double*>(sel_smem);                       // [R][D]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qs + SEL_ROWS * D);        // [R][256]
  uint64_t* keys = reinterpret_cast<uint64_t*>(hist + SEL_ROWS * 256);    // [R][c_stride]

  const int HbWb = p.Hb * p.Wb;
  const int bh = blockIdx.z;
  const int b = bh / p.H;
  const int tq = blockIdx.y;
  const int sp0 = blockIdx.x * SEL_ROWS;
  const int nrows = min(SEL_ROWS, HbWb - sp0);
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  const int64_t m_first = begin >> 1;               // oldest cached block (absolute)
  const int slot0 = static_cast<int>(m_first % p.cap_blk);
  const int nKT = static_cast<int>((end >> 1) - m_first);
  const int tq_kv = nKT - p.nQT + tq;               // query time step in the key timeline
  const int ncand = (tq_kv + 1) * HbWb;             // causal candidates
  const int nQB = p.nQT * HbWb;
  const int tid = threadIdx.x;

  // Pull every candidate's pooled key row toward L2 up front, so the scoring
  // loop below waits on L2 rather than on DRAM (rows are D*8 bytes).
  {
    constexpr int LINES = D * 8 / 128;
    for (int e = tid; e < ncand * LINES; e += SEL_THREADS) {
      const int j = e / LINES, l = e % LINES;
      const int tk = j / HbWb, spk = j - tk * HbWb;
      const int slot = (slot0 + tk) % p.cap_blk;
      const double* line = p.k_pool + ((static_cast<int64_t>(bh) * p.cap_blk + slot) * HbWb + spk) * D + l * 16;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(line));
    }
  }

  const double* qsrc = p.q_pool + (static_cast<int64_t>(bh) * nQB + tq * HbWb + sp0) * D;
  for (int e = tid; e < SEL_ROWS * D; e += SEL_THREADS)
    qs[e] = e < nrows * D ? qsrc[e] : 0.0;

  int y0[SEL_ROWS], y1[SEL_ROWS], x0[SEL_ROWS], x1[SEL_ROWS];
#pragma unroll
  for (int r = 0; r < SEL_ROWS; ++r) {
    const int sp = min(sp0 + r, HbWb - 1);
    window_bounds(sp / p.Wb, p.Hb, p.window, p.window_mode, y0[r], y1[r]);
    window_bounds(sp % p.Wb, p.Wb, p.window, p.window_mode, x0[r], x1[r]);
  }
  __syncthreads();

  // Phase 1: keys of all causal candidates for the CTA's rows.
  const double2* q2 = reinterpret_cast<const double2*>(qs);
  for (int j = tid; j < ncand; j += SEL_THREADS) {
    const int tk = j / HbWb, spk = j - tk * HbWb;
    const int yk = spk / p.Wb, xk = spk - yk * p.Wb;
    const int slot = (slot0 + tk) % p.cap_blk;
    const double2* kr = reinterpret_cast<const double2*>(
        p.k_pool + ((static_cast<int64_t>(bh) * p.cap_blk + slot) * HbWb + spk) * D);
    double s[SEL_ROWS];
#pragma unroll
    for (int r = 0; r < SEL_ROWS; ++r) s[r] = 0.0;
#pragma unroll 16
    for (int c2 = 0; c2 < D / 2; ++c2) {
      const double2 kv = __ldg(kr + c2);
#pragma unroll
      for (int r = 0; r < SEL_ROWS; ++r) {
        const double2 qv = q2[r * (D / 2) + c2];
        s[r] = __dadd_rn(s[r], __dmul_rn(qv.x, kv.x));
        s[r] = __dadd_rn(s[r], __dmul_rn(qv.y, kv.y));
      }
    }
#pragma unroll
    for (int r = 0; r < SEL_ROWS; ++r) {
      if (r < nrows) {
        const bool ok = yk >= y0[r] && yk < y1[r] && xk >= x0[r] && xk < x1[r];
        // adding +0.0 turns -0.0 into +0.0, so equal scores get equal keys
        const double sc = __dadd_rn(__ddiv_rn(s[r], p.sqrt_d), 0.0);
        keys[r * p.c_stride + j] = ok ? order_key(sc) : 0ull;
      }
    }
  }
  __syncthreads();

  // Phase 2: one warp per query block.
  const int r = tid >> 5;
  if (r >= nrows) return;
  const int lane = tid & 31;
  int wy0, wy1, wx0, wx1;
  window_bounds((sp0 + r) / p.Wb, p.Hb, p.window, p.window_mode, wy0, wy1);
  window_bounds((sp0 + r) % p.Wb, p.Wb, p.window, p.window_mode, wx0, wx1);
  const int C = (tq_kv + 1) * (wy1 - wy0) * (wx1 - wx0);
  int K;
  if (p.top_k > 0) {
    K = min(C, p.top_k);
  } else {
    const double kd = ceil(__dmul_rn(p.density, static_cast<double>(C)));
    K = min(C, max(1, static_cast<int>(kd)));
  }
  const uint64_t* krow = keys + r * p.c_stride;
  uint32_t* h = hist + r * 256;

  // Exact K-th largest key, 8 bits at a time from the top.
  uint64_t prefix = 0, pmask = 0;
  int krem = K;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) h[i] = 0u;
    __syncwarp();
    for (int j = lane; j < ncand; j += 32) {
      const uint64_t key = krow[j];
      if (key != 0ull && (key & pmask) == prefix)
        atomicAdd(&h[static_cast<int>((key >> shift) & 255u)], 1u);
    }
    __syncwarp();
    uint32_t c[8];
    int local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = h[8 * lane + i];
      local += static_cast<int>(c[i]);
    }
    int suf = local;  // keys of this prefix whose digit falls in bins >= 8*lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += v;
    }
    const int above_lane = suf - local;
    const uint32_t hit = __ballot_sync(0xffffffffu, above_lane < krem && suf >= krem);
    const int src = __ffs(hit) - 1;
    int digit = 0, knew = 0;
    if (lane == src) {
      int acc = above_lane;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (acc + static_cast<int>(c[i]) >= krem) {
          digit = 8 * lane + i;
          knew = krem - acc;
          break;
        }
        acc += static_cast<int>(c[i]);
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, src);
    krem = __shfl_sync(0xffffffffu, knew, src);
    prefix |= static_cast<uint64_t>(digit) << shift;
    pmask |= static_cast<uint64_t>(255) << shift;
    __syncwarp();
  }
  const double tau = key_value(prefix);
  const uint64_t k_hi = order_key(__dadd_rn(tau, p.tie_eps));
  const uint64_t k_lo = order_key(__dsub_rn(tau, p.tie_eps));
  int above = 0;
  for (int j = lane; j < ncand; j += 32) above += krow[j] > k_hi ? 1 : 0;
  above = __reduce_add_sync(0xffffffffu, above);
  const int need = K - above;

  const int64_t row = static_cast<int64_t>(bh) * nQB + tq * HbWb + sp0 + r;
  int32_t* out = p.blk_idx + row * p.kmax;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int n_band = 0, n_sel = 0;
  for (int j0 = 0; j0 < ncand; j0 += 32) {
    const int j = j0 + lane;
    const uint64_t key = j < ncand ? krow[j] : 0ull;
    const bool in_above = key > k_hi;
    const bool in_band = key >= k_lo && key <= k_hi;
    const uint32_t band_mask = __ballot_sync(0xffffffffu, in_band);
    const bool take = in_above || (in_band && (n_band + __popc(band_mask & lt_mask)) < need);
    const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = n_sel + __popc(take_mask & lt_mask);
      if (pos < p.kmax) out[pos] = j;
      else atomicOr(p.err, DEVERR_BOUNDS);
    }
    n_band += __popc(band_mask);
    n_sel += __popc(take_mask);
  }
  for (int pos = K + lane; pos < p.kmax; pos += 32) out[pos] = -1;
  if (lane == 0) p.blk_cnt[row] = K;
}

}  // namespace lcsa
