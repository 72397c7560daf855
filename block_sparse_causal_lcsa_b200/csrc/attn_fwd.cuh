// Sparse attention over the kept block pairs (FlashVSR summary, section 2.2
// stage 2: "apply full attention within the selected regions"), on the
// 5th-generation tensor cores of sm_100a.
//
// One CTA computes one 128-token query block of one (stream, head) against
// its K_i kept key blocks, with an online softmax:
//   warp 0      TMA producer: the Q tile once, then K and V tiles of each kept
//               block into two 3-stage rings (5-D tensor maps over
//               (d, x, y, frame, stream*head); one box = one frame of a block
//               = 64 tokens x 64 channels, 128-byte swizzled). A K stage is
//               released as soon as S_j has consumed it, a V stage once PV_j
//               has, so loads run up to three blocks ahead.
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//               accumulators (128 lanes x 128 fp32 columns), then
//               O += P_j V_j with P_j read from tensor memory and V_j from
//               shared memory. S_{j+1} is issued before PV_j, so the tensor
//               core computes the next scores while the softmax runs.
//   warps 2-5   softmax warpgroup, one query row per thread (= TMEM lane):
//               tcgen05.ld of S_j, mask the missing frame of a one-frame
//               block, running max with lazy rescaling of O (only when the
//               max grows by more than 2^8), P = 2^(s*log2e/sqrt(d) - m) on
//               the special-function unit, rounded to bf16 and stored with
//               tcgen05.st over the first 64 columns of S_j; row sums in
//               fp32; at the end O / l to bf16 and the log-sum-exp.
// Tensor memory: 512 columns (S0 | S1 | O). Shared memory for D = 128:
// Q 32 KB + K 3x32 KB + V 3x32 KB = 224 KB, one CTA per SM.
// Every wait is bounded; on a timeout the CTA drains its in-flight copies and
// MMAs, frees its tensor memory and exits with the error word set.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int KV_STAGES = 3;

template <int D>
struct AttnLayout {
  static constexpr int TILE_BYTES = 128 * D * 2;   // 128 tokens x D bf16
  static constexpr int CHUNK_BYTES = 128 * 128;    // 128 rows x 64 channels (one swizzle column)
  static constexpr int BOX_BYTES = 64 * 128;       // one frame of a block, 64 channels
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KV_STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + KV_STAGES * TILE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
};

// mbarrier slots
enum : int {
  B_Q_FULL = 0,
  B_K_FULL = 1,                        // KV_STAGES
  B_K_EMPTY = B_K_FULL + KV_STAGES,    // KV_STAGES
  B_V_FULL = B_K_EMPTY + KV_STAGES,    // KV_STAGES
  B_V_EMPTY = B_V_FULL + KV_STAGES,    // KV_STAGES
  B_S_FULL = B_V_EMPTY + KV_STAGES,    // 2 TMEM buffers
  B_P_FULL = B_S_FULL + 2,             // 2
  B_PV_DONE = B_P_FULL + 2,            // 2
  B_DRAIN = B_PV_DONE + 2,
  B_COUNT = B_DRAIN + 1
};

constexpr int ATTN_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O_COL = 256;

struct AttnParams {
  const int32_t* blk_idx;    // [B*H][nQB][kmax]
  const int32_t* blk_cnt;    // [B*H][nQB]
  __nv_bfloat16* o;
  float* lse;                // [B*H][Tq][Y][X] or null
  int64_t osh, ost, osy, osx;  // strides of o (stream stride = H * osh)
  int32_t H, Tq, Y, X, Hb, Wb, nQT, nQB, kmax, cap;
  float scale_log2;          // log2(e) / sqrt(D)
  uint64_t wait_limit_ns;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

// Warp-uniform bounded wait: every lane polls, all lanes agree on the result.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = wait_bounded(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_test(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return;
  }
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A (M x 16, bf16 pairs per 32-bit column)
// from tensor memory, one 128xNx16 step issued by one thread.
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  using L = AttnLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::OFF_BAR;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * B_COUNT + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // CTA -> (stream*head, query block); within a head the query blocks of the
  // newest time step (the longest rows) go first.
  const int HbWb = p.Hb * p.Wb;
  const int bh = blockIdx.x / p.nQB;
  const int rr = blockIdx.x % p.nQB;
  const int tq = p.nQT - 1 - rr / HbWb;
  const int sp = rr % HbWb;
  const int b = bh / p.H;
  const int yq = sp / p.Wb, xq = sp % p.Wb;
  const int64_t row = static_cast<int64_t>(bh) * p.nQB + tq * HbWb + sp;
  const int32_t* blist = p.blk_idx + row * p.kmax;
  int n = p.blk_cnt[row];
  if (n < 0 || n > p.kmax) {
    if (threadIdx.x == 0) atomicOr(p.err, DEVERR_BOUNDS);
    n = 0;
  }
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  const int64_t m_first = begin >> 1;
  const int nkb = static_cast<int>((end >> 1) - m_first) * HbWb;  // valid block ids
  const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;   // older frame of the query block (-1: missing)

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(bar(i), (i == B_P_FULL || i == B_P_FULL + 1) ? 128u : 1u);
    *abort_flag = 0;
    mbar_init_fence();
    tma_prefetch_map(&tmQ);
    tma_prefetch_map(&tmK);
    tma_prefetch_map(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx w{p.wait_limit_ns, abort_flag, p.err};

  auto checked = [&](int blk) -> int {
    if (blk < 0 || blk >= nkb) {
      atomicOr(p.err, DEVERR_BOUNDS);
      blk = 0;
    }
    return blk;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      auto load_tile = [&](const CUtensorMap* map, uint32_t dst, uint32_t bar_full, int x8, int y8,
                           int fr0, int fr1) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_5d(dst + c * L::CHUNK_BYTES, map, bar_full, c * 64, x8, y8, fr0, bh);
          tma_load_5d(dst + c * L::CHUNK_BYTES + L::BOX_BYTES, map, bar_full, c * 64, x8, y8, fr1, bh);
        }
      };
      mbar_arrive_expect_tx(bar(B_Q_FULL), L::TILE_BYTES);
      // a missing older query frame is replaced by the newer one (rows not stored)
      load_tile(&tmQ, sbase + L::OFF_Q, bar(B_Q_FULL), 8 * xq, 8 * yq, fq0 < 0 ? fq0 + 1 : fq0, fq0 + 1);
      int issued_k = 0, issued_v = 0;
      int next_blk = checked(blist[0]);
      for (int j = 0; j < n; ++j) {
        const int blk = next_blk;
        if (j + 1 < n) next_blk = checked(blist[j + 1]);
        const int st = j % KV_STAGES;
        const uint32_t ph = ((j / KV_STAGES) - 1) & 1;
        const int tk = blk / HbWb, spk = blk % HbWb;
        const int64_t m = m_first + tk;
        const int64_t a1 = 2 * m + 1;
        const int64_t a0 = (2 * m < begin) ? a1 : 2 * m;   // one-frame block: load its frame twice
        const int s0 = static_cast<int>(a0 % p.cap), s1 = static_cast<int>(a1 % p.cap);
        const int x8 = 8 * (spk % p.Wb), y8 = 8 * (spk / p.Wb);
        if (j >= KV_STAGES && !wait_bounded(bar(B_K_EMPTY + st), ph, w)) break;
        mbar_arrive_expect_tx(bar(B_K_FULL + st), L::TILE_BYTES);
        load_tile(&tmK, sbase + L::OFF_K + st * L::TILE_BYTES, bar(B_K_FULL + st), x8, y8, s0, s1);
        issued_k = j + 1;
        if (j >= KV_STAGES && !wait_bounded(bar(B_V_EMPTY + st), ph, w)) break;
        mbar_arrive_expect_tx(bar(B_V_FULL + st), L::TILE_BYTES);
        load_tile(&tmV, sbase + L::OFF_V + st * L::TILE_BYTES, bar(B_V_FULL + st), x8, y8, s0, s1);
        issued_v = j + 1;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA goes away
        drain_wait(bar(B_Q_FULL), 0, w.limit_ns);
        for (int j = issued_k > KV_STAGES ? issued_k - KV_STAGES : 0; j < issued_k; ++j)
          drain_wait(bar(B_K_FULL + j % KV_STAGES), (j / KV_STAGES) & 1, w.limit_ns);
        for (int j = issued_v > KV_STAGES ? issued_v - KV_STAGES : 0; j < issued_v; ++j)
          drain_wait(bar(B_V_FULL + j % KV_STAGES), (j / KV_STAGES) & 1, w.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, true);
      auto issue_s = [&](int j) -> bool {
        const int ks = j % KV_STAGES;
        if (!wait_bounded(bar(B_K_FULL + ks), (j / KV_STAGES) & 1, w)) return false;
        tc_fence_after();
        const uint32_t qa = sbase + L::OFF_Q;
        const uint32_t ka = sbase + L::OFF_K + ks * L::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // K-major operands: 16 channels = 32 bytes inside a 128-byte swizzled row
          const uint32_t off = (kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32;
          umma_ss(tmem + (j & 1) * 128, desc_sw128(qa + off, 16, 1024),
                  desc_sw128(ka + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_S_FULL + (j & 1)));
        umma_commit(bar(B_K_EMPTY + ks));
        return true;
      };
      bool ok = wait_bounded(bar(B_Q_FULL), 0, w);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int sb = j & 1;
        const int vs = j % KV_STAGES;
        // S_{j+1} overwrites the TMEM buffer of P_{j-1}; PV_{j-1} was issued
        // before it and tcgen05 MMAs of one thread execute in order.
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;
        if (!(ok = wait_bounded(bar(B_P_FULL + sb), (j >> 1) & 1, w))) break;
        if (!(ok = wait_bounded(bar(B_V_FULL + vs), (j / KV_STAGES) & 1, w))) break;
        tc_fence_after();
        const uint32_t va = sbase + L::OFF_V + vs * L::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = P (16 keys = 8 packed columns of S_j's TMEM buffer); B = V
          // (MN-major: channels contiguous), 16 keys = 16 rows of 128 bytes,
          // 64-channel columns 16 KB apart.
          umma_ts(tmem + TMEM_O_COL, tmem + sb * 128 + kk * 8,
                  desc_sw128(va + kk * 2048, L::CHUNK_BYTES, 1024), ID_PV,
                  (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_PV_DONE + sb));
        umma_commit(bar(B_V_EMPTY + vs));
      }
      // no MMA may still be running when the tensor memory is released
      umma_commit(bar(B_DRAIN));
      drain_wait(bar(B_DRAIN), 0, w.limit_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;                 // TMEM lanes [32*quarter, +32)
    const int r = quarter * 32 + lane;            // query row of the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool oldest_partial = (begin & 1) != 0; // the oldest cached block has one frame
    const float scale = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;         // running max (log2 units) and sum
    bool done = n > 0;
    int next_blk = n > 0 ? checked(blist[0]) : 0;
    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      const bool partial = oldest_partial && next_blk < HbWb;
      if (j + 1 < n) next_blk = checked(blist[j + 1]);
      if (!warp_wait(bar(B_S_FULL + sb), (j >> 1) & 1, w)) { done = false; break; }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld_32x32b_x32(t_lane + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(t_lane + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_32x32b_x32(t_lane + sb * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
      tmem_ld_32x32b_x32(t_lane + sb * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
      tmem_ld_wait();
      if (partial) {
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        mx0 = fmaxf(mx0, __uint_as_float(s[c]));
        mx1 = fmaxf(mx1, __uint_as_float(s[c + 1]));
      }
      const float mx = fmaxf(mx0, mx1) * scale;   // scale > 0: max commutes with it
      float m_new = m_run;
      if (j == 0 || mx > m_run + 8.f) m_new = mx;
      if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
        // O may only be rescaled once PV_{j-1} has finished
        if (!warp_wait(bar(B_PV_DONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1, w)) { done = false; break; }
        tc_fence_after();
        const float alpha = ex2_approx(m_run - m_new);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld_32x32b_x32(t_lane + TMEM_O_COL + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st_32x32b_x32(t_lane + TMEM_O_COL + c0, o);
        }
        tmem_st_wait();
        l_run *= alpha;
      }
      m_run = m_new;
      const float neg_m = -m_run;
      uint32_t pk[64];
      float sum0 = 0.f, sum1 = 0.f, sum2 = 0.f, sum3 = 0.f;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(s[2 * c]), scale, neg_m));
        const float p1 = ex2_approx(fmaf(__uint_as_float(s[2 * c + 1]), scale, neg_m));
        const float p2 = ex2_approx(fmaf(__uint_as_float(s[2 * c + 2]), scale, neg_m));
        const float p3 = ex2_approx(fmaf(__uint_as_float(s[2 * c + 3]), scale, neg_m));
        sum0 += p0;
        sum1 += p1;
        sum2 += p2;
        sum3 += p3;
        pk[c] = pack_bf16x2(p0, p1);
        pk[c + 1] = pack_bf16x2(p2, p3);
      }
      l_run += (sum0 + sum1) + (sum2 + sum3);
      // P_j over the first 64 columns of S_j's buffer (S_j has been read)
      tmem_st_32x32b_x32(t_lane + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st_32x32b_x32(t_lane + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL + sb));
    }
    if (done) done = warp_wait(bar(B_PV_DONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1, w);
    const bool row_valid = !(fq0 < 0 && r < 64);
    const int f = r >> 6, yy = (r >> 3) & 7, xx = r & 7;
    const int frame = fq0 + f;
    const int y = 8 * yq + yy, x = 8 * xq + xx;
    __nv_bfloat16* orow = p.o + static_cast<int64_t>(bh) * p.osh + static_cast<int64_t>(frame) * p.ost +
                          static_cast<int64_t>(y) * p.osy + static_cast<int64_t>(x) * p.osx;
    if (done) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(t_lane + TMEM_O_COL + c0, o);
        tmem_ld_wait();
        uint32_t ob[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          ob[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(ob[4 * k], ob[4 * k + 1], ob[4 * k + 2], ob[4 * k + 3]);
        }
      }
      if (p.lse != nullptr && row_valid)
        p.lse[((static_cast<int64_t>(bh) * p.Tq + frame) * p.Y + y) * p.X + x] =
            (m_run + log2f(l_run)) * 0.69314718055994531f;
    } else if (n == 0 && row_valid) {
      // no kept block (cannot happen for selections made by this library)
      uint4* dst = reinterpret_cast<uint4*>(orow);
      for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
      if (p.lse != nullptr)
        p.lse[((static_cast<int64_t>(bh) * p.Tq + frame) * p.Y + y) * p.X + x] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace lcsa
