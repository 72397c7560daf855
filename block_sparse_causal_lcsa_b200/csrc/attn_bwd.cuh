// Gradients of the sparse attention over the kept block pairs, for training
// with the block-sparse causal mask (FlashVSR summary, section 2.2 stage 2:
// the full-attention model is adapted to block-sparse causal attention and
// trained with the flow-matching loss; stage 3 trains the one-step student
// with the same mask). The selection is a constant of the backward pass.
//
// With S = Q K^T / sqrt(D), P = exp(S - LSE) (the forward's log-sum-exp),
// dP = dO V^T, delta_r = sum_d dO_rd O_rd and dS = P (dP - delta):
//   dQ = dS K / sqrt(D),  dK = dS^T Q / sqrt(D),  dV = P^T dO.
// Four kernels, deterministic (no floating-point atomics):
//   bwd_prep_kernel   per query block: delta and LSE*log2(e) of its 128 rows in
//                     block order (rows of a missing older frame get LSE = +inf
//                     and delta = 0, so they contribute nothing below).
//   bwd_lists_kernel  per key block: the query blocks that kept it, ascending
//                     (the transpose of the selection), one warp per key block.
//   bwd_dq_kernel     one CTA per query block over its kept key blocks: S and
//                     dP (tcgen05, shared-memory operands) into tensor memory,
//                     dS in bf16 into its own tensor-memory columns, dQ += dS K
//                     (dS from tensor memory) issued after the next block's S
//                     and dP so that it overlaps the next elementwise step.
//   bwd_dkdv_kernel   one CTA per key block over the query blocks that kept
//                     it: S^T = K Q^T and dP^T = V dO^T, P^T and dS^T in bf16
//                     written back over them, dV += P^T dO and dK += dS^T Q, both
//                     accumulated in tensor memory.
// Six warps per CTA: a TMA producer, a single-thread MMA issuer and four
// elementwise warps (one tile row per thread = TMEM lane), as in the forward.
// Every wait is bounded; on a timeout a CTA drains, frees its tensor memory
// and exits with the error word set.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int BWD_THREADS = 192;
constexpr int BWD_EW_THREADS = 128;
constexpr float LOG2E = 1.4426950408889634f;

struct BwdParams {
  const int32_t* blk_idx;     // [B*H][nQB][kmax]
  const int32_t* blk_cnt;     // [B*H][nQB]
  const __nv_bfloat16* o;     // like q
  const __nv_bfloat16* d_o;   // like q
  const float* lse;           // [B*H][Tq][Y][X]
  __nv_bfloat16* dq;          // like q (own strides)
  __nv_bfloat16* dk;          // cache layout [B][H][cap][Y][X][D], contiguous
  __nv_bfloat16* dv;
  float* lse2_blk;            // workspace [B*H][nQB][128]
  float* delta_blk;           // workspace [B*H][nQB][128]
  int32_t* qcnt;              // workspace [B*H][nKBmax]
  int32_t* qlist;             // workspace [B*H][nKBmax][nQB]
  int64_t osh, ost, osy, osx;       // strides of o
  int64_t gsh, gst, gsy, gsx;       // strides of d_o
  int64_t qsh, qst, qsy, qsx;       // strides of dq
  int32_t BH, H, Tq, Y, X, Hb, Wb, nQT, nQB, kmax, cap, nKBmax;
  float scale_log2;           // log2(e) / sqrt(D)
  float scale;                // 1 / sqrt(D)
  uint64_t wait_limit_ns;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

// ---------------------------------------------------------------- prep
// One CTA of 128 threads per query block; thread r owns row r of the block
// (frame r/64 of the block, y = (r/8)%8, x = r%8).
template <int D>
__global__ void __launch_bounds__(128) bwd_prep_kernel(const __grid_constant__ BwdParams p) {
  const int unit = blockIdx.x;                       // bh * nQB + query block
  const int bh = unit / p.nQB, qb = unit % p.nQB;
  const int HbWb = p.Hb * p.Wb;
  const int tq = qb / HbWb, sp = qb % HbWb;
  const int r = threadIdx.x;
  const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;
  const int frame = fq0 + (r >> 6);
  float lse2 = INFINITY, delta = 0.f;
  if (frame >= 0) {
    const int y = 8 * (sp / p.Wb) + ((r >> 3) & 7), x = 8 * (sp % p.Wb) + (r & 7);
    const uint4* orow = reinterpret_cast<const uint4*>(p.o + bh * p.osh + frame * p.ost + y * p.osy + x * p.osx);
    const uint4* grow = reinterpret_cast<const uint4*>(p.d_o + bh * p.gsh + frame * p.gst + y * p.gsy + x * p.gsx);
    uint4 ov[D / 8], gv[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      ov[c] = __ldg(orow + c);
      gv[c] = __ldg(grow + c);
    }
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&ov[c]);
      const __nv_bfloat162* g = reinterpret_cast<const __nv_bfloat162*>(&gv[c]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fa = __bfloat1622float2(a[k]), fg = __bfloat1622float2(g[k]);
        acc = fmaf(fa.x, fg.x, acc);
        acc = fmaf(fa.y, fg.y, acc);
      }
    }
    delta = acc;
    lse2 = p.lse[((static_cast<int64_t>(bh) * p.Tq + frame) * p.Y + y) * p.X + x] * LOG2E;
  }
  p.lse2_blk[static_cast<int64_t>(unit) * 128 + r] = lse2;
  p.delta_blk[static_cast<int64_t>(unit) * 128 + r] = delta;
}

// ---------------------------------------------------------------- lists
// One warp per (stream*head, key block): lanes test 32 query blocks at a time
// (binary search in the query block's ascending kept list) and a ballot
// appends the hits in ascending order.
__global__ void __launch_bounds__(256) bwd_lists_kernel(const __grid_constant__ BwdParams p) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(p.BH) * p.nKBmax) return;
  const int bh = static_cast<int>(wid / p.nKBmax), jk = static_cast<int>(wid % p.nKBmax);
  int32_t* out = p.qlist + wid * p.nQB;
  int n = 0;
  for (int i0 = 0; i0 < p.nQB; i0 += 32) {
    const int i = i0 + lane;
    bool hit = false;
    if (i < p.nQB) {
      const int64_t row = static_cast<int64_t>(bh) * p.nQB + i;
      int lo = 0, hi = min(max(p.blk_cnt[row], 0), p.kmax);
      const int32_t* bl = p.blk_idx + row * p.kmax;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int v = bl[mid];
        if (v < jk) lo = mid + 1;
        else hi = mid;
      }
      hit = lo < min(max(p.blk_cnt[row], 0), p.kmax) && bl[lo] == jk;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    if (hit) out[n + __popc(m & ((1u << lane) - 1u))] = i;
    n += __popc(m);
  }
  if (lane == 0) p.qcnt[wid] = n;
}

// Bounded waits shared by the two MMA kernels (same contract as the forward).
__device__ __forceinline__ bool bwd_warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = wait_bounded(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void bwd_drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}
// D[tmem] (+)= A[tmem] * B[smem]: A (128 x 16 bf16, two per 32-bit column) from tensor memory.
__device__ __forceinline__ void bwd_umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D>
struct BwdLayout {
  static constexpr int TILE = 128 * D * 2;       // 128 tokens x D bf16
  static constexpr int CHUNK = 128 * 128;        // 128 rows x 64 channels (one swizzle column)
  static constexpr int BOX = 64 * 128;           // one frame of a block, 64 channels
  // dq kernel: Q, dO resident; K and V rings of 2
  static constexpr int DQ_Q = 0, DQ_DO = TILE, DQ_K = 2 * TILE, DQ_V = 4 * TILE, DQ_BAR = 6 * TILE;
  // dkdv kernel: K, V resident; Q, dO rings of 2, plus the 128 LSE and delta values of each stage
  static constexpr int KV_K = 0, KV_V = TILE, KV_Q = 2 * TILE, KV_DO = 4 * TILE, KV_VEC = 6 * TILE;
  static constexpr int KV_BAR = KV_VEC + 2 * 1024;
  static constexpr int SMEM_DQ = DQ_BAR + 256 + 1024;
  static constexpr int SMEM_KV = KV_BAR + 256 + 1024;
};

// Ring slots of a key block's two frames (a one-frame block loads its frame
// twice). The host passes begin in [0, cap), so the frame numbers lie in
// [0, 2 cap) and a slot is a conditional subtract; 32-bit arithmetic only.
__device__ __forceinline__ void bwd_key_coords(const BwdParams& p, int b, int blk, int& x8, int& y8, int& s0,
                                               int& s1) {
  const int HbWb = p.Hb * p.Wb;
  const int begin = static_cast<int>(p.kv_begin[b]);
  const int tk = blk / HbWb, spk = blk - tk * HbWb;
  const int a1 = 2 * ((begin >> 1) + tk) + 1;
  const int a0 = a1 - 1 < begin ? a1 : a1 - 1;
  s0 = a0 >= p.cap ? a0 - p.cap : a0;
  s1 = a1 >= p.cap ? a1 - p.cap : a1;
  const int yb = spk / p.Wb;
  x8 = 8 * (spk - yb * p.Wb);
  y8 = 8 * yb;
}

template <int D>
__device__ __forceinline__ void bwd_load_tile(const CUtensorMap* map, uint32_t dst, uint32_t bar, int x8, int y8,
                                              int fr0, int fr1, int bh) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    tma_load_5d(dst + c * BwdLayout<D>::CHUNK, map, bar, c * 64, x8, y8, fr0, bh);
    tma_load_5d(dst + c * BwdLayout<D>::CHUNK + BwdLayout<D>::BOX, map, bar, c * 64, x8, y8, fr1, bh);
  }
}

// Elementwise step of one 128x128 tile, one row per thread: P = 2^(S*scale_log2
// - lse2), G = P (dP - delta), both rounded to bf16; P is written back in place
// over the first 64 columns of S and G to the 64 columns at t_g (t_g = t_dp
// writes it in place too: column chunk c of 32 values packs into columns
// [16c, 16c+16), which chunk c has already read). The column vectors lse2 /
// delta (or per-row scalars) and the masks come from the caller.
template <bool COL_VECTORS>
__device__ __forceinline__ void bwd_tile_elementwise(uint32_t t_s, uint32_t t_dp, uint32_t t_g, float scale_log2,
                                                     const float* lse2v, const float* deltav, float lse2_row,
                                                     float delta_row, bool zero_cols_lo, bool zero_row,
                                                     bool write_p) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t s[32], dp[32];
    tmem_ld_32x32b_x32(t_s + c * 32, s);
    tmem_ld_32x32b_x32(t_dp + c * 32, dp);
    tmem_ld_wait();
    uint32_t pp[16], gg[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float pv[2], gv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = c * 32 + 2 * k + h;
        const float l2 = COL_VECTORS ? lse2v[col] : lse2_row;
        const float dl = COL_VECTORS ? deltav[col] : delta_row;
        float pe = ex2_approx(fmaf(__uint_as_float(s[2 * k + h]), scale_log2, -l2));
        if (zero_row || (zero_cols_lo && col < 64)) pe = 0.f;
        pv[h] = pe;
        gv[h] = pe * (__uint_as_float(dp[2 * k + h]) - dl);
      }
      pp[k] = pack_bf16x2(pv[0], pv[1]);
      gg[k] = pack_bf16x2(gv[0], gv[1]);
    }
    if (write_p) tmem_st_32x32b_x16(t_s + c * 16, pp);
    tmem_st_32x32b_x16(t_g + c * 16, gg);
  }
  tmem_st_wait();
}

// ---------------------------------------------------------------- dQ
constexpr uint32_t DS_COL = 256;   // dS (bf16 pairs, 64 columns) of the dQ kernel
constexpr uint32_t DQ_COL = 384;   // dQ accumulator of the dQ kernel
enum : int {
  DQB_QD_FULL = 0,      // Q and dO of the block
  DQB_K_FULL = 1,       // 2
  DQB_K_EMPTY = 3,      // 2
  DQB_V_FULL = 5,       // 2
  DQB_V_EMPTY = 7,      // 2
  DQB_SD_FULL = 9,      // S and dP of the current kept block
  DQB_G_FULL = 10,      // dS written (128 arrivals)
  DQB_DQ_DONE = 11,     // dQ MMA of the current kept block
  DQB_DRAIN = 12,
  DQB_COUNT = 13
};

template <int D>
__global__ void __launch_bounds__(BWD_THREADS, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
              const __grid_constant__ BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::DQ_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::DQ_BAR + 8 * DQB_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::DQ_BAR + 8 * DQB_COUNT + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int HbWb = p.Hb * p.Wb;
  const int unit = blockIdx.x;
  const int bh = unit / p.nQB, qb = unit % p.nQB;
  const int b = bh / p.H;
  const int tq = qb / HbWb, sp = qb % HbWb;
  const int yq = sp / p.Wb, xq = sp % p.Wb;
  const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;
  const int64_t row = static_cast<int64_t>(bh) * p.nQB + qb;
  const int32_t* blist = p.blk_idx + row * p.kmax;
  int n = p.blk_cnt[row];
  if (n < 0 || n > p.kmax) {
    if (threadIdx.x == 0) atomicOr(p.err, DEVERR_BOUNDS);
    n = 0;
  }
  const int64_t begin = p.kv_begin[b];
  const int nkb = static_cast<int>((p.kv_end[b] >> 1) - (begin >> 1)) * HbWb;

  if (threadIdx.x == 0) {
    for (int i = 0; i < DQB_COUNT; ++i) mbar_init(bar(i), i == DQB_G_FULL ? BWD_EW_THREADS : 1u);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;          // S: cols 0-127, dP: 128-255, dS: 256-319, dQ: 384-511
  const WaitCtx w{p.wait_limit_ns, abort_flag, p.err};
  auto checked = [&](int blk) -> int {
    if (blk < 0 || blk >= nkb) {
      atomicOr(p.err, DEVERR_BOUNDS);
      blk = 0;
    }
    return blk;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(bar(DQB_QD_FULL), 2 * L::TILE);
      const int f0 = fq0 < 0 ? fq0 + 1 : fq0;  // a missing older frame: load the newer one twice
      bwd_load_tile<D>(&tmQ, sbase + L::DQ_Q, bar(DQB_QD_FULL), 8 * xq, 8 * yq, f0, fq0 + 1, bh);
      bwd_load_tile<D>(&tmDO, sbase + L::DQ_DO, bar(DQB_QD_FULL), 8 * xq, 8 * yq, f0, fq0 + 1, bh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        int x8, y8, s0, s1;
        bwd_key_coords(p, b, checked(blist[j]), x8, y8, s0, s1);
        const int st = j & 1;
        if (j >= 2) {
          if (!wait_bounded(bar(DQB_K_EMPTY + st), ((j >> 1) - 1) & 1, w)) break;
          if (!wait_bounded(bar(DQB_V_EMPTY + st), ((j >> 1) - 1) & 1, w)) break;
        }
        mbar_arrive_expect_tx(bar(DQB_K_FULL + st), L::TILE);
        bwd_load_tile<D>(&tmK, sbase + L::DQ_K + st * L::TILE, bar(DQB_K_FULL + st), x8, y8, s0, s1, bh);
        mbar_arrive_expect_tx(bar(DQB_V_FULL + st), L::TILE);
        bwd_load_tile<D>(&tmV, sbase + L::DQ_V + st * L::TILE, bar(DQB_V_FULL + st), x8, y8, s0, s1, bh);
        issued = j + 1;
      }
      if (*abort_flag) {
        bwd_drain_wait(bar(DQB_QD_FULL), 0, w.limit_ns);
        for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j) {
          bwd_drain_wait(bar(DQB_K_FULL + (j & 1)), (j >> 1) & 1, w.limit_ns);
          bwd_drain_wait(bar(DQB_V_FULL + (j & 1)), (j >> 1) & 1, w.limit_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t ID_SS = idesc_bf16_f32(128, 128, false);   // S, dP: K-major A and B
      constexpr uint32_t ID_DQ = idesc_bf16_f32(128, D, true);      // dQ: B = K, channels contiguous
      bool ok = wait_bounded(bar(DQB_QD_FULL), 0, w);
      // dQ += dS K for block j-1 (dS in its own tensor-memory columns) is issued
      // right after S_j and dP_j, so it runs while the elementwise warps work on
      // block j.
      auto issue_dq = [&](int jj) {
        // one descriptor per operand; a step's is the base plus its byte offset / 16
        const uint64_t kd = desc_sw128(sbase + L::DQ_K + (jj & 1) * L::TILE, L::CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = dS (16 keys = 8 packed columns), B = K: 16 keys = 16 rows of 128 bytes,
          // 64-channel columns 16 KB apart
          bwd_umma_ts(tmem + DQ_COL, tmem + DS_COL + kk * 8, kd + kk * (2048 >> 4), ID_DQ,
                      (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(DQB_DQ_DONE));
        umma_commit(bar(DQB_K_EMPTY + (jj & 1)));
      };
      for (int j = 0; ok && j < n; ++j) {
        const int st = j & 1;
        if (!(ok = wait_bounded(bar(DQB_K_FULL + st), (j >> 1) & 1, w))) break;
        if (!(ok = wait_bounded(bar(DQB_V_FULL + st), (j >> 1) & 1, w))) break;
        // S_j and dP_j overwrite what the elementwise warps read for block j-1
        if (j > 0 && !(ok = wait_bounded(bar(DQB_G_FULL), (j - 1) & 1, w))) break;
        tc_fence_after();
        const uint64_t qd = desc_sw128(sbase + L::DQ_Q, 16, 1024), od = desc_sw128(sbase + L::DQ_DO, 16, 1024);
        const uint64_t kd = desc_sw128(sbase + L::DQ_K + st * L::TILE, 16, 1024);
        const uint64_t vd = desc_sw128(sbase + L::DQ_V + st * L::TILE, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * L::CHUNK + (kk & 3) * 32) >> 4;
          umma_ss(tmem, qd + off16, kd + off16, ID_SS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * L::CHUNK + (kk & 3) * 32) >> 4;
          umma_ss(tmem + 128, od + off16, vd + off16, ID_SS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(DQB_SD_FULL));
        umma_commit(bar(DQB_V_EMPTY + st));
        if (j > 0) issue_dq(j - 1);
      }
      if (ok && (ok = wait_bounded(bar(DQB_G_FULL), (n - 1) & 1, w))) {
        tc_fence_after();
        issue_dq(n - 1);
      }
      umma_commit(bar(DQB_DRAIN));
      bwd_drain_wait(bar(DQB_DRAIN), 0, w.limit_ns);
    }
  } else {
    // ---------------------------------------------------------- elementwise, row = query
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float lse2 = p.lse2_blk[row * 128 + r];
    const float delta = p.delta_blk[row * 128 + r];
    const bool oldest_partial = (begin & 1) != 0;
    bool done = n > 0;
    for (int j = 0; j < n; ++j) {
      const bool partial = oldest_partial && checked(blist[j]) < HbWb;  // keys 0-63 absent
      if (!bwd_warp_wait(bar(DQB_SD_FULL), j & 1, w)) { done = false; break; }
      // the dS columns are free once dQ of block j-1 (their last reader) is done
      if (j > 0 && !bwd_warp_wait(bar(DQB_DQ_DONE), (j - 1) & 1, w)) { done = false; break; }
      tc_fence_after();
      bwd_tile_elementwise<false>(t_lane, t_lane + 128, t_lane + DS_COL, p.scale_log2, nullptr, nullptr, lse2, delta,
                                  partial, false, false);
      tc_fence_before();
      mbar_arrive(bar(DQB_G_FULL));
    }
    if (done) done = bwd_warp_wait(bar(DQB_DQ_DONE), (n - 1) & 1, w);
    const bool row_valid = !(fq0 < 0 && r < 64);
    const int frame = fq0 + (r >> 6);
    const int y = 8 * yq + ((r >> 3) & 7), x = 8 * xq + (r & 7);
    __nv_bfloat16* drow = p.dq + bh * p.qsh + static_cast<int64_t>(frame) * p.qst + y * p.qsy + x * p.qsx;
    if (row_valid && (done || n == 0)) {
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t g[32];
        if (n > 0) {
          tmem_ld_32x32b_x32(t_lane + DQ_COL + c0, g);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) g[k] = 0u;
        }
        uint4* dst = reinterpret_cast<uint4*>(drow + c0);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(g[8 * k]) * p.scale, __uint_as_float(g[8 * k + 1]) * p.scale);
          v.y = pack_bf16x2(__uint_as_float(g[8 * k + 2]) * p.scale, __uint_as_float(g[8 * k + 3]) * p.scale);
          v.z = pack_bf16x2(__uint_as_float(g[8 * k + 4]) * p.scale, __uint_as_float(g[8 * k + 5]) * p.scale);
          v.w = pack_bf16x2(__uint_as_float(g[8 * k + 6]) * p.scale, __uint_as_float(g[8 * k + 7]) * p.scale);
          dst[k] = v;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- dK, dV
enum : int {
  KVB_KV_FULL = 0,      // K and V of the key block
  KVB_Q_FULL = 1,       // 2 stages: Q, dO, LSE and delta of a query block
  KVB_Q_EMPTY = 3,      // 2
  KVB_SD_FULL = 5,      // S^T and dP^T
  KVB_G_FULL = 6,       // P^T and dS^T written (128 arrivals)
  KVB_ACC_DONE = 7,     // dV and dK MMAs of the current query block
  KVB_DRAIN = 8,
  KVB_COUNT = 9
};

template <int D>
__global__ void __launch_bounds__(BWD_THREADS, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + L::KV_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::KV_BAR + 8 * KVB_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::KV_BAR + 8 * KVB_COUNT + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int HbWb = p.Hb * p.Wb;
  const int bh = blockIdx.x / p.nKBmax, jk = blockIdx.x % p.nKBmax;
  const int b = bh / p.H;
  const int64_t begin = p.kv_begin[b];
  const int nkb = static_cast<int>((p.kv_end[b] >> 1) - (begin >> 1)) * HbWb;
  if (jk >= nkb) return;   // this stream has fewer key blocks (whole CTA, before any barrier)
  const int64_t lrow = static_cast<int64_t>(bh) * p.nKBmax + jk;
  const int32_t* qlist = p.qlist + lrow * p.nQB;
  int n = p.qcnt[lrow];
  if (n < 0 || n > p.nQB) {
    if (threadIdx.x == 0) atomicOr(p.err, DEVERR_BOUNDS);
    n = 0;
  }
  const bool key_partial = (begin & 1) != 0 && jk < HbWb;   // key rows 0-63 absent

  if (threadIdx.x == 0) {
    for (int i = 0; i < KVB_COUNT; ++i) mbar_init(bar(i), i == KVB_G_FULL ? BWD_EW_THREADS : 1u);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;          // S^T 0-127, dP^T 128-255, dV 256-383, dK 384-511
  const WaitCtx w{p.wait_limit_ns, abort_flag, p.err};
  auto checked_q = [&](int i) -> int {
    if (i < 0 || i >= p.nQB) {
      atomicOr(p.err, DEVERR_BOUNDS);
      i = 0;
    }
    return i;
  };

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0 && n > 0) {
      int x8, y8, s0, s1;
      bwd_key_coords(p, b, jk, x8, y8, s0, s1);
      mbar_arrive_expect_tx(bar(KVB_KV_FULL), 2 * L::TILE);
      bwd_load_tile<D>(&tmK, sbase + L::KV_K, bar(KVB_KV_FULL), x8, y8, s0, s1, bh);
      bwd_load_tile<D>(&tmV, sbase + L::KV_V, bar(KVB_KV_FULL), x8, y8, s0, s1, bh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int qb = checked_q(qlist[j]);
        const int tq = qb / HbWb, sp = qb % HbWb;
        const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;
        const int f0 = fq0 < 0 ? fq0 + 1 : fq0;
        const int st = j & 1;
        if (j >= 2 && !wait_bounded(bar(KVB_Q_EMPTY + st), ((j >> 1) - 1) & 1, w)) break;
        const uint32_t fb = bar(KVB_Q_FULL + st);
        mbar_arrive_expect_tx(fb, 2 * L::TILE + 1024);
        bwd_load_tile<D>(&tmQ, sbase + L::KV_Q + st * L::TILE, fb, 8 * (sp % p.Wb), 8 * (sp / p.Wb), f0, fq0 + 1, bh);
        bwd_load_tile<D>(&tmDO, sbase + L::KV_DO + st * L::TILE, fb, 8 * (sp % p.Wb), 8 * (sp / p.Wb), f0, fq0 + 1, bh);
        const int64_t u = static_cast<int64_t>(bh) * p.nQB + qb;
        bulk_load(sbase + L::KV_VEC + st * 1024, p.lse2_blk + u * 128, 512, fb);
        bulk_load(sbase + L::KV_VEC + st * 1024 + 512, p.delta_blk + u * 128, 512, fb);
        issued = j + 1;
      }
      if (*abort_flag) {
        bwd_drain_wait(bar(KVB_KV_FULL), 0, w.limit_ns);
        for (int j = issued > 2 ? issued - 2 : 0; j < issued; ++j)
          bwd_drain_wait(bar(KVB_Q_FULL + (j & 1)), (j >> 1) & 1, w.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t ID_SS = idesc_bf16_f32(128, 128, false);   // S^T, dP^T: K-major A and B
      constexpr uint32_t ID_ACC = idesc_bf16_f32(128, D, true);     // dV, dK: B channels contiguous
      bool ok = wait_bounded(bar(KVB_KV_FULL), 0, w);
      for (int j = 0; ok && j < n; ++j) {
        const int st = j & 1;
        if (!(ok = wait_bounded(bar(KVB_Q_FULL + st), (j >> 1) & 1, w))) break;
        // S^T and dP^T overwrite the buffers the previous dV / dK MMAs read
        if (j > 0 && !(ok = wait_bounded(bar(KVB_ACC_DONE), (j - 1) & 1, w))) break;
        tc_fence_after();
        const uint32_t qa = sbase + L::KV_Q + st * L::TILE, ga = sbase + L::KV_DO + st * L::TILE;
        // one descriptor per operand; a step's is the base plus its byte offset / 16
        const uint64_t kd = desc_sw128(sbase + L::KV_K, 16, 1024), vd = desc_sw128(sbase + L::KV_V, 16, 1024);
        const uint64_t qd = desc_sw128(qa, 16, 1024), gd = desc_sw128(ga, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * L::CHUNK + (kk & 3) * 32) >> 4;
          umma_ss(tmem, kd + off16, qd + off16, ID_SS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * L::CHUNK + (kk & 3) * 32) >> 4;
          umma_ss(tmem + 128, vd + off16, gd + off16, ID_SS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(KVB_SD_FULL));
        if (!(ok = wait_bounded(bar(KVB_G_FULL), j & 1, w))) break;
        tc_fence_after();
        const uint64_t gdm = desc_sw128(ga, L::CHUNK, 1024), qdm = desc_sw128(qa, L::CHUNK, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // dV += P^T dO and dK += dS^T Q: A (16 queries = 8 packed columns) from tensor
          // memory; B = dO / Q, 16 queries = 16 rows of 128 bytes, 64-channel columns 16 KB apart
          bwd_umma_ts(tmem + 256, tmem + kk * 8, gdm + kk * (2048 >> 4), ID_ACC, (j > 0 || kk > 0) ? 1u : 0u);
          bwd_umma_ts(tmem + 384, tmem + 128 + kk * 8, qdm + kk * (2048 >> 4), ID_ACC, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(KVB_ACC_DONE));
        umma_commit(bar(KVB_Q_EMPTY + st));
      }
      umma_commit(bar(KVB_DRAIN));
      bwd_drain_wait(bar(KVB_DRAIN), 0, w.limit_ns);
    }
  } else {
    // ---------------------------------------------------------- elementwise, row = key
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool zero_row = key_partial && r < 64;
    bool done = true;
    for (int j = 0; j < n; ++j) {
      const int st = j & 1;
      // the stage's LSE / delta vectors (bulk-copied with Q and dO), then S^T and dP^T
      if (!bwd_warp_wait(bar(KVB_Q_FULL + st), (j >> 1) & 1, w)) { done = false; break; }
      if (!bwd_warp_wait(bar(KVB_SD_FULL), j & 1, w)) { done = false; break; }
      tc_fence_after();
      const float* vec = reinterpret_cast<const float*>(smem + L::KV_VEC + st * 1024);
      bwd_tile_elementwise<true>(t_lane, t_lane + 128, t_lane + 128, p.scale_log2, vec, vec + 128, 0.f, 0.f, false,
                                 zero_row, true);
      tc_fence_before();
      mbar_arrive(bar(KVB_G_FULL));
    }
    if (done && n > 0) done = bwd_warp_wait(bar(KVB_ACC_DONE), (n - 1) & 1, w);
    int x8, y8, s0, s1;
    bwd_key_coords(p, b, jk, x8, y8, s0, s1);
    const int slot = (r >> 6) ? s1 : s0;
    const int64_t tok = ((static_cast<int64_t>(bh) * p.cap + slot) * p.Y + y8 + ((r >> 3) & 7)) * p.X + x8 + (r & 7);
    if (!zero_row && (done || n == 0)) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {          // dV, then dK (scaled)
        __nv_bfloat16* dst_row = (which == 0 ? p.dv : p.dk) + tok * D;
        const float sc = which == 0 ? 1.f : p.scale;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t g[32];
          if (n > 0) {
            tmem_ld_32x32b_x32(t_lane + 256 + which * 128 + c0, g);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) g[k] = 0u;
          }
          uint4* dst = reinterpret_cast<uint4*>(dst_row + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(g[8 * k]) * sc, __uint_as_float(g[8 * k + 1]) * sc);
            v.y = pack_bf16x2(__uint_as_float(g[8 * k + 2]) * sc, __uint_as_float(g[8 * k + 3]) * sc);
            v.z = pack_bf16x2(__uint_as_float(g[8 * k + 4]) * sc, __uint_as_float(g[8 * k + 5]) * sc);
            v.w = pack_bf16x2(__uint_as_float(g[8 * k + 6]) * sc, __uint_as_float(g[8 * k + 7]) * sc);
            dst[k] = v;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace lcsa
