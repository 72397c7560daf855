// Coarse block map, causal and locality masks, and top-K selection
// (FlashVSR summary, section 2.2 stage 2: coarse block-to-block attention map,
// keep the top-K block pairs, causal masking; section 2.3: a spatial window
// per query with a boundary-truncate or boundary-preserve rule).
//
// Two kernels, joined by a caller-provided workspace of 64-bit keys
// [rows][c_stride]:
// score_kernel  one CTA per (16 query blocks) x (32 candidate key blocks) of a
//   (stream, head, temporal block). The 16 pooled query rows and the 32 pooled
//   key rows are staged in shared memory (key rows padded to D+1 doubles so
//   the 32 lanes of a warp, each reading its own row, hit distinct banks);
//   each thread scores one candidate against 4 rows - 4 independent float64
//   chains, each summed in channel order with every product rounded before it
//   is added (no fused multiply-add), then divided by sqrt(D): the same
//   float64 value as the definition, bit for bit. Scores are stored as
//   order-preserving 64-bit keys; candidates outside the row's window get
//   key 0, below every finite score.
// topk_warp_kernel  one warp per query block, the row's keys held in
//   registers (at most 2048 causal candidates): the exact K-th largest key by
//   a 1-bit radix select (one warp-wide count per bit from the top, stopping
//   once a single key matches), then one ascending pass keeps every block
//   above tau+eps and the lowest-index blocks of the band [tau-eps, tau+eps].
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int SC_ROWS = 16;       // query blocks per score CTA
constexpr int SC_CANDS = 32;      // candidate key blocks per score CTA
constexpr int SC_THREADS = 128;   // 32 candidates x 4 groups of 4 rows

struct SelectParams {
  const double* q_pool;   // [B][H][nQT][Hb][Wb][D]
  const double* k_pool;   // ring [B][H][cap_blk][Hb][Wb][D]
  uint64_t* keys;         // workspace [B*H*nQB][c_stride]
  int32_t* blk_idx;       // [B][H][nQT*Hb*Wb][kmax]
  int32_t* blk_cnt;       // [B][H][nQT*Hb*Wb]
  int32_t B, H, Hb, Wb, nQT, cap_blk;
  int32_t top_k, window, window_mode, kmax;
  int32_t c_stride;       // row stride (keys) of the workspace = most causal candidates of any row
  double density, tie_eps, sqrt_d;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

__host__ __device__ constexpr size_t score_smem_bytes(int D) {
  return sizeof(double) * (static_cast<size_t>(SC_ROWS) * D + static_cast<size_t>(SC_CANDS) * (D + 2));
}

__device__ __forceinline__ uint64_t order_key(double s) {
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(s));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(uint64_t k) {
  const uint64_t u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double(static_cast<long long>(u));
}

// Window of key blocks along one axis (n blocks) seen from query block i.
// Modes 0 / 1: w blocks centred on the block, truncated / preserved at the
// edge. Modes 2 / 3: the blocks holding a token that some token of block i
// sees through its w-token window (truncated / preserved).
__host__ __device__ __forceinline__ void window_bounds(int i, int n, int w, int mode, int& lo, int& hi) {
  if (w <= 0) { lo = 0; hi = n; return; }
  if (mode >= 2) {
    int a, b, c, d;
    token_window(8 * i, 8 * n, w, mode, a, b);
    token_window(8 * i + 7, 8 * n, w, mode, c, d);
    lo = a / 8;
    hi = (d - 1) / 8 + 1;
    return;
  }
  const int r = w / 2;
  if (mode == 0) {  // truncate at the frame edge
    lo = i - r > 0 ? i - r : 0;
    hi = i + r + 1 < n ? i + r + 1 : n;
  } else {          // preserve: shift inward, keep w blocks
    int st = i - r < n - w ? i - r : n - w;
    lo = st > 0 ? st : 0;
    hi = lo + w < n ? lo + w : n;
  }
}

// Candidate range of a stream: the key timeline's oldest cached block and the
// query time step tq's position in it.
struct StreamGeom {
  int64_t m_first;  // absolute index of the oldest cached block
  int slot0;        // its ring slot
  int tq_kv;        // key temporal block of query temporal block tq
  int ncand;        // causal candidates (tq_kv + 1) * Hb * Wb
};

__device__ __forceinline__ StreamGeom stream_geom(const SelectParams& p, int b, int tq) {
  StreamGeom g;
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  g.m_first = begin >> 1;
  // the host passes begin in [0, cap), so the oldest block's slot is its index
  g.slot0 = static_cast<int>(g.m_first);
  const int nKT = static_cast<int>((end >> 1) - g.m_first);
  g.tq_kv = nKT - p.nQT + tq;
  g.ncand = (g.tq_kv + 1) * p.Hb * p.Wb;
  return g;
}

template <int D>
__global__ void __launch_bounds__(SC_THREADS)
score_kernel(const __grid_constant__ SelectParams p) {
  extern __shared__ __align__(16) double sc_smem[];
  double* qs = sc_smem;                         // [SC_ROWS][D]
  // candidate rows padded to D + 2 doubles: 16-byte aligned for paired loads,
  // and lanes (one candidate each) 4 banks apart, so a quarter warp's 16-byte
  // loads hit distinct banks
  double* ks = qs + SC_ROWS * D;                // [SC_CANDS][D+2]

  const int HbWb = p.Hb * p.Wb;
  const int nQB = p.nQT * HbWb;
  const int bh = blockIdx.z / p.nQT;
  const int tq = blockIdx.z % p.nQT;
  const int b = bh / p.H;
  const int sp0 = blockIdx.y * SC_ROWS;
  const int nrows = min(SC_ROWS, HbWb - sp0);
  const StreamGeom g = stream_geom(p, b, tq);
  const int c0 = blockIdx.x * SC_CANDS;
  if (c0 >= g.ncand || nrows <= 0) return;
  const int ncur = min(SC_CANDS, g.ncand - c0);
  const int tid = threadIdx.x;

  // With a window, most (row, candidate) pairs of a CTA can lie outside every
  // row's window: a CTA none of whose pairs is inside only writes key 0.
  if (p.window > 0) {
    bool any = false;
    const int cand = tid % SC_CANDS;
    if (cand < ncur) {
      const int spk = (c0 + cand) % HbWb;
      const int yk = spk / p.Wb, xk = spk - yk * p.Wb;
      for (int r = tid / SC_CANDS; r < nrows; r += SC_THREADS / SC_CANDS) {
        const int sp = sp0 + r;
        int y0, y1, x0, x1;
        window_bounds(sp / p.Wb, p.Hb, p.window, p.window_mode, y0, y1);
        window_bounds(sp % p.Wb, p.Wb, p.window, p.window_mode, x0, x1);
        any |= yk >= y0 && yk < y1 && xk >= x0 && xk < x1;
      }
    }
    if (!__syncthreads_or(any)) {
      for (int e = tid; e < nrows * SC_CANDS; e += SC_THREADS) {
        const int r = e / SC_CANDS, c = e % SC_CANDS;
        if (c < ncur)
          p.keys[(static_cast<int64_t>(bh) * nQB + tq * HbWb + sp0 + r) * p.c_stride + c0 + c] = 0ull;
      }
      return;
    }
  }

  const int warp = tid >> 5, lane = tid & 31;
  constexpr int V2 = D / 2;                       // 16-byte vectors per pooled row
  constexpr int PER_LANE = V2 / 32;               // vectors per lane per row
  constexpr int ROWS_PER_WARP = SC_CANDS / (SC_THREADS / 32);
  // query rows: warp w stages rows w, w+4, ... (plain copy, zero beyond nrows)
  const double2* qsrc = reinterpret_cast<const double2*>(
      p.q_pool + (static_cast<int64_t>(bh) * nQB + tq * HbWb + sp0) * D);
#pragma unroll
  for (int rr = warp; rr < SC_ROWS; rr += SC_THREADS / 32) {
#pragma unroll
    for (int v = 0; v < PER_LANE; ++v) {
      const int e = v * 32 + lane;
      const double2 x = rr < nrows ? __ldg(qsrc + rr * V2 + e) : make_double2(0.0, 0.0);
      qs[rr * D + 2 * e] = x.x;
      qs[rr * D + 2 * e + 1] = x.y;
    }
  }
  // candidate rows: warp w stages ROWS_PER_WARP consecutive rows, all loads issued before
  // any store so that the L2 round trips overlap
  double2 buf[ROWS_PER_WARP][PER_LANE];
#pragma unroll
  for (int i = 0; i < ROWS_PER_WARP; ++i) {
    const int cc = warp * ROWS_PER_WARP + i;
    const int j = c0 + cc;
    if (cc < ncur) {
      const int tk = j / HbWb, spk = j - tk * HbWb;
      const int slot = g.slot0 + tk < p.cap_blk ? g.slot0 + tk : g.slot0 + tk - p.cap_blk;
      const double2* src = reinterpret_cast<const double2*>(
          p.k_pool + ((static_cast<int64_t>(bh) * p.cap_blk + slot) * HbWb + spk) * D);
#pragma unroll
      for (int v = 0; v < PER_LANE; ++v) buf[i][v] = __ldg(src + v * 32 + lane);
    } else {
#pragma unroll
      for (int v = 0; v < PER_LANE; ++v) buf[i][v] = make_double2(0.0, 0.0);
    }
  }
#pragma unroll
  for (int i = 0; i < ROWS_PER_WARP; ++i) {
    const int cc = warp * ROWS_PER_WARP + i;
#pragma unroll
    for (int v = 0; v < PER_LANE; ++v) {
      const int e = v * 32 + lane;
      reinterpret_cast<double2*>(ks + cc * (D + 2))[e] = buf[i][v];
    }
  }
  __syncthreads();

  const int cc = tid % SC_CANDS;
  const int r0 = (tid / SC_CANDS) * 4;
  if (cc >= ncur) return;
  const double2* kr = reinterpret_cast<const double2*>(ks + cc * (D + 2));
  const double2* q0 = reinterpret_cast<const double2*>(qs + (r0 + 0) * D);
  const double2* q1 = reinterpret_cast<const double2*>(qs + (r0 + 1) * D);
  const double2* q2 = reinterpret_cast<const double2*>(qs + (r0 + 2) * D);
  const double2* q3 = reinterpret_cast<const double2*>(qs + (r0 + 3) * D);
  double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
  // channel pairs (c, c + 1) loaded together; the products are still added
  // one channel at a time, in channel order
#pragma unroll 2
  for (int c2 = 0; c2 < D / 2; ++c2) {
    const double2 kv = kr[c2];
    const double2 a = q0[c2], b = q1[c2], cq = q2[c2], dq = q3[c2];
    s0 = __dadd_rn(s0, __dmul_rn(a.x, kv.x));
    s1 = __dadd_rn(s1, __dmul_rn(b.x, kv.x));
    s2 = __dadd_rn(s2, __dmul_rn(cq.x, kv.x));
    s3 = __dadd_rn(s3, __dmul_rn(dq.x, kv.x));
    s0 = __dadd_rn(s0, __dmul_rn(a.y, kv.y));
    s1 = __dadd_rn(s1, __dmul_rn(b.y, kv.y));
    s2 = __dadd_rn(s2, __dmul_rn(cq.y, kv.y));
    s3 = __dadd_rn(s3, __dmul_rn(dq.y, kv.y));
  }
  const int j = c0 + cc;
  int yk = 0, xk = 0;
  if (p.window > 0) {
    const int spk = j % HbWb;
    yk = spk / p.Wb;
    xk = spk - yk * p.Wb;
  }
  const double sv[4] = {s0, s1, s2, s3};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + i;
    if (r >= nrows) break;
    const int sp = sp0 + r;
    bool ok = true;   // without a window every causal candidate is allowed
    if (p.window > 0) {
      int y0, y1, x0, x1;
      window_bounds(sp / p.Wb, p.Hb, p.window, p.window_mode, y0, y1);
      window_bounds(sp % p.Wb, p.Wb, p.window, p.window_mode, x0, x1);
      ok = yk >= y0 && yk < y1 && xk >= x0 && xk < x1;
    }
    // adding +0.0 turns -0.0 into +0.0, so equal scores get equal keys
    const double sc = __dadd_rn(__ddiv_rn(sv[i], p.sqrt_d), 0.0);
    const int64_t row = static_cast<int64_t>(bh) * nQB + tq * HbWb + sp;
    p.keys[row * p.c_stride + j] = ok ? order_key(sc) : 0ull;
  }
}

// One warp per query block (4 per CTA): the row's keys sit in registers as
// 32-bit halves (candidate j = 32*i + lane in slot i, at most 32*KPL
// candidates). The K-th largest key is found one bit at a time, first over
// the high halves, then - only if several keys share the K-th largest high
// half - over the low halves of those keys; a bit's count is one compare per
// slot and lane and one warp-wide add, with no barrier.
constexpr int TKW_WARPS = 4;
template <int KPL>
__global__ void __launch_bounds__(TKW_WARPS * 32)
topk_warp_kernel(const __grid_constant__ SelectParams p) {
  const int HbWb = p.Hb * p.Wb;
  const int nQB = p.nQT * HbWb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row64 = static_cast<int64_t>(blockIdx.x) * TKW_WARPS + warp;
  if (row64 >= static_cast<int64_t>(p.B) * p.H * nQB) return;
  const int row = static_cast<int>(row64);   // rows < 2^31 (checked on the host)
  const int bh = row / nQB;
  const int qi = row - bh * nQB;
  const int tq = qi / HbWb, sp = qi - tq * HbWb;
  const StreamGeom g = stream_geom(p, bh / p.H, tq);
  const int ncand = g.ncand;
  if (ncand > 32 * KPL) {
    if (lane == 0) atomicOr(p.err, DEVERR_BOUNDS);
    return;
  }
  int y0 = 0, y1 = p.Hb, x0 = 0, x1 = p.Wb;
  if (p.window > 0) {
    window_bounds(sp / p.Wb, p.Hb, p.window, p.window_mode, y0, y1);
    window_bounds(sp % p.Wb, p.Wb, p.window, p.window_mode, x0, x1);
  }
  const int C = (g.tq_kv + 1) * (y1 - y0) * (x1 - x0);
  int K;
  if (p.top_k > 0) {
    K = min(C, p.top_k);
  } else {
    const double kd = ceil(__dmul_rn(p.density, static_cast<double>(C)));
    K = min(C, max(1, static_cast<int>(kd)));
  }
  const uint64_t* krow = p.keys + static_cast<int64_t>(row) * p.c_stride;
  const int nslots = (ncand + 31) / 32;
  uint32_t hi[KPL], lo[KPL];
  int lc = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    const int j = 32 * i + lane;
    const uint64_t k = (i < nslots && j < ncand) ? krow[j] : 0ull;
    hi[i] = static_cast<uint32_t>(k >> 32);
    lo[i] = static_cast<uint32_t>(k);
    lc += k != 0ull;                           // window-masked candidates (key 0) are not ranked
  }
  // nact: unmasked keys that match the prefix found so far. A masked key has
  // no bit set, so it never matches a prefix extended by a set bit and is
  // never counted.
  int nact = __reduce_add_sync(0xffffffffu, lc);
  int krem = K;
  uint32_t phi = 0, plo = 0;
  int bit = 31;
  for (; bit >= 0 && nact > 1; --bit) {
    const uint32_t t = (phi >> bit) | 1u;
    lc = 0;
#pragma unroll
    for (int i = 0; i < KPL; ++i)
      if (i < nslots) lc += (hi[i] >> bit) == t;
    const int cnt = __reduce_add_sync(0xffffffffu, lc);
    if (cnt >= krem) {
      nact = cnt;
      phi |= 1u << bit;
    } else {
      krem -= cnt;
      nact -= cnt;
    }
  }
  // bits of the high half above hbit are decided (all of them when hbit = -1)
  const int hbit = bit;
  int lbit = 32;
  if (nact > 1) {
    // several keys share the K-th largest high half: rank their low halves
    for (bit = 31; bit >= 0 && nact > 1; --bit) {
      const uint32_t t = (plo >> bit) | 1u;
      lc = 0;
#pragma unroll
      for (int i = 0; i < KPL; ++i)
        if (i < nslots) lc += hi[i] == phi && (lo[i] >> bit) == t;
      const int cnt = __reduce_add_sync(0xffffffffu, lc);
      if (cnt >= krem) {
        nact = cnt;
        plo |= 1u << bit;
      } else {
        krem -= cnt;
        nact -= cnt;
      }
    }
    lbit = bit;
  }
  uint64_t kth = (static_cast<uint64_t>(phi) << 32) | plo;
  if (lbit >= 0) {
    // a single unmasked key matches the decided bits: it is the K-th largest
    uint32_t fh = 0, fl = 0;
    bool have = false;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
      if (i >= nslots) break;
      const bool nz = (hi[i] | lo[i]) != 0u;
      bool m;
      if (lbit == 32) {
        m = nz && (hbit + 1 >= 32 || (hi[i] >> (hbit + 1)) == (phi >> (hbit + 1)));
      } else {
        m = hi[i] == phi && (lbit + 1 >= 32 || (lo[i] >> (lbit + 1)) == (plo >> (lbit + 1)));
      }
      if (m) {
        fh = hi[i];
        fl = lo[i];
        have = true;
      }
    }
    const uint32_t who = __ballot_sync(0xffffffffu, have);
    if (who != 0u) {
      const int src = __ffs(who) - 1;
      kth = (static_cast<uint64_t>(__shfl_sync(0xffffffffu, fh, src)) << 32) | __shfl_sync(0xffffffffu, fl, src);
    }
  }
  const double tau = key_value(kth);
  const uint64_t k_hi = order_key(__dadd_rn(tau, p.tie_eps));
  const uint64_t k_lo = order_key(__dsub_rn(tau, p.tie_eps));
  lc = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i)
    if (i < nslots) lc += ((static_cast<uint64_t>(hi[i]) << 32) | lo[i]) > k_hi;
  const int need = K - __reduce_add_sync(0xffffffffu, lc);
  int32_t* out = p.blk_idx + static_cast<int64_t>(row) * p.kmax;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int n_band = 0, n_sel = 0;
#pragma unroll
  for (int i = 0; i < KPL; ++i) {
    if (i >= nslots) break;
    const int j = 32 * i + lane;
    const uint64_t k = (static_cast<uint64_t>(hi[i]) << 32) | lo[i];
    const bool in_above = k > k_hi;
    const bool in_band = k >= k_lo && k <= k_hi;
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
