// Coarse block map, causal and locality masks, and top-K selection
// (FlashVSR summary, section 2.2 stage 2: coarse block-to-block attention map,
// keep the top-K block pairs, causal masking; section 2.3: a spatial window
// per query with a boundary-truncate or boundary-preserve rule).
//
// One CTA (8 warps) owns 8 query blocks of one (stream, head, temporal block)
// and all of their causal candidates. Phase 1 stages 32 pooled key rows at a
// time in shared memory and computes every (query, candidate) score with its
// own thread, in channel order, each product rounded before it is added
// (no fused multiply-add), then divides by sqrt(D): the same float64 value as
// the definition, bit for bit. Phase 2 gives each warp one query block: the
// K-th largest allowed score is found exactly by a 64-step radix search on the
// order-preserving integer image of the doubles (warp ballots and reductions),
// then one ascending pass keeps every block above tau+eps plus the
// lowest-index blocks of the band [tau-eps, tau+eps].
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int SEL_ROWS = 8;       // query blocks per CTA (one warp each in phase 2)
constexpr int SEL_TILE = 32;      // candidates per staged tile
constexpr int SEL_THREADS = SEL_ROWS * 32;

struct SelectParams {
  const double* q_pool;   // [B][H][nQT][Hb][Wb][D]
  const double* k_pool;   // ring [B][H][cap_blk][Hb][Wb][D]
  int32_t* blk_idx;       // [B][H][nQT*Hb*Wb][kmax]
  int32_t* blk_cnt;       // [B][H][nQT*Hb*Wb]
  int32_t H, D, Hb, Wb, nQT, cap_blk;
  int32_t top_k, window, window_mode, kmax;
  int32_t c_stride;       // row stride (doubles) of the score buffer in shared memory
  double density, tie_eps, sqrt_d;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

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

__global__ void __launch_bounds__(SEL_THREADS)
select_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) double sm[];
  const int D = p.D;
  double* qs = sm;                                   // [SEL_ROWS][D]
  double* ks = qs + SEL_ROWS * D;                    // [SEL_TILE][D+1]
  double* sc = ks + SEL_TILE * (D + 1);              // [SEL_ROWS][c_stride]

  const int HbWb = p.Hb * p.Wb;
  const int bh = blockIdx.z;
  const int b = bh / p.H;
  const int tq = blockIdx.y;
  const int sp0 = blockIdx.x * SEL_ROWS;
  const int nrows = min(SEL_ROWS, HbWb - sp0);
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  const int64_t m_first = begin >> 1;               // oldest cached block (absolute)
  const int nKT = static_cast<int>((end >> 1) - m_first);
  const int tq_kv = nKT - p.nQT + tq;               // query time step in the key timeline
  const int ncand = (tq_kv + 1) * HbWb;             // causal candidates
  const int nQB = p.nQT * HbWb;
  const int tid = threadIdx.x;

  for (int e = tid; e < SEL_ROWS * D; e += SEL_THREADS) {
    const int r = e / D, c = e % D;
    qs[e] = r < nrows ? p.q_pool[((static_cast<int64_t>(bh) * nQB) + tq * HbWb + sp0 + r) * D + c]
                      : 0.0;
  }

  // Phase 1: scores of all causal candidates.
  const int my_r = tid >> 5, my_j = tid & 31;
  for (int j0 = 0; j0 < ncand; j0 += SEL_TILE) {
    __syncthreads();
    for (int e = tid; e < SEL_TILE * D; e += SEL_THREADS) {
      const int jj = e / D, c = e % D;
      const int j = j0 + jj;
      double v = 0.0;
      if (j < ncand) {
        const int tk = j / HbWb, spk = j % HbWb;
        const int64_t slot = (m_first + tk) % p.cap_blk;
        v = p.k_pool[((static_cast<int64_t>(bh) * p.cap_blk + slot) * HbWb + spk) * D + c];
      }
      ks[jj * (D + 1) + c] = v;
    }
    __syncthreads();
    const int j = j0 + my_j;
    if (my_r < nrows && j < ncand) {
      const double* qr = qs + my_r * D;
      const double* kr = ks + my_j * (D + 1);
      double s = 0.0;
      for (int c = 0; c < D; ++c) s = __dadd_rn(s, __dmul_rn(qr[c], kr[c]));
      sc[my_r * p.c_stride + j] = __ddiv_rn(s, p.sqrt_d);
    }
  }
  __syncthreads();

  // Phase 2: one warp per query block.
  const int r = my_r;
  if (r >= nrows) return;
  const int lane = my_j;
  const int sp = sp0 + r;
  const int yq = sp / p.Wb, xq = sp % p.Wb;
  int y0, y1, x0, x1;
  window_bounds(yq, p.Hb, p.window, p.window_mode, y0, y1);
  window_bounds(xq, p.Wb, p.window, p.window_mode, x0, x1);
  const int C = (tq_kv + 1) * (y1 - y0) * (x1 - x0);
  int K;
  if (p.top_k > 0) {
    K = min(C, p.top_k);
  } else {
    const double kd = ceil(__dmul_rn(p.density, static_cast<double>(C)));
    K = min(C, max(1, static_cast<int>(kd)));
  }
  // Replace this row's scores by their order-preserving keys; blocks outside
  // the window get key 0, below every finite score.
  uint64_t* krow = reinterpret_cast<uint64_t*>(sc + r * p.c_stride);
  for (int j = lane; j < ncand; j += 32) {
    const int spk = j % HbWb;
    const int yk = spk / p.Wb, xk = spk % p.Wb;
    const bool ok = yk >= y0 && yk < y1 && xk >= x0 && xk < x1;
    // adding +0.0 turns -0.0 into +0.0, so equal scores get equal keys
    const double s = __dadd_rn(reinterpret_cast<const double*>(krow)[j], 0.0);
    krow[j] = ok ? order_key(s) : 0ull;
  }
  __syncwarp();

  // Exact K-th largest key: the largest t with #{key >= t} >= K.
  uint64_t T = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const uint64_t cand = T | (1ull << bit);
    int cnt = 0;
    for (int j = lane; j < ncand; j += 32) cnt += krow[j] >= cand ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= K) T = cand;
  }
  const double tau = key_value(T);
  const uint64_t k_hi = order_key(__dadd_rn(tau, p.tie_eps));
  const uint64_t k_lo = order_key(__dsub_rn(tau, p.tie_eps));
  int above = 0;
  for (int j = lane; j < ncand; j += 32) above += krow[j] > k_hi ? 1 : 0;
  above = __reduce_add_sync(0xffffffffu, above);
  const int need = K - above;

  const int64_t row = static_cast<int64_t>(bh) * nQB + tq * HbWb + sp;
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
