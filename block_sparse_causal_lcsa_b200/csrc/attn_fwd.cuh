// Sparse attention over the kept block pairs (FlashVSR summary, section 2.2
// stage 2: "apply full attention within the selected regions"), on the
// 5th-generation tensor cores of sm_100a.
//
// One CTA computes one 128-token query block of one (stream, head) against
// its K_i kept key blocks, with an online softmax. Seven warps:
//   warps 0, 6  TMA producers: warp 0 loads the Q tile once and the K tile of
//               each kept block, warp 6 the V tiles, into two 3-stage rings
//               (5-D tensor maps over (d, x, y, frame, stream*head); one box =
//               one frame of a block = 64 tokens x 64 channels, 128-byte
//               swizzled). A K stage is released as soon as S_j has consumed
//               it (the S_j barrier), a V stage once PV_j has (the PV_j
//               barrier); separate producers let the K loads run ahead of the
//               V stages the softmax holds up.
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into one of THREE TMEM
//               score buffers (128 lanes x 128 fp32 columns each), then
//               O += P_j V_j with P_j read from tensor memory. Scores run two
//               blocks ahead of the softmax: S_{j+2} is issued before PV_j, as
//               soon as PV_{j-1} has completed (it overwrites the buffer P_{j-1}
//               was read from; MMAs into different accumulators are not ordered
//               with respect to each other). Issuing S_{j+2} after PV_j
//               instead put the issue of PV_j on the softmax's critical path.
//               The PV barriers are one per score buffer: with two (by parity)
//               and this order, the final wait for PV_{n-1} could match a phase
//               of PV_{n-3} that had not completed yet.
//   warps 2-5   softmax warpgroup, one query row per thread (= TMEM lane):
//               tcgen05.ld of S_j, mask the missing frame of a one-frame
//               block, running max with lazy rescaling of O (only when the
//               max grows by more than 2^8), P = 2^(s*log2e/sqrt(d) - m) with
//               packed fp32x2 arithmetic - exponentials on the
//               special-function unit (sending some of them to a polynomial
//               on the FMA pipe measured slower here) - rounded to bf16 pairs
//               by one cvt.rn.bf16x2.f32 per pair (fewer instructions than
//               rounding with integer ops, and measured faster: the softmax
//               loop is bound by its instruction issue as much as by the
//               special-function unit) and
//               stored with tcgen05.st over the first 64 columns of S_j's
//               buffer; row sums in fp32; at the end O / l in bf16 and the
//               log-sum-exp.
// Tensor memory: 512 columns (S0 | S1 | S2 | O). Shared memory for D = 128:
// Q 32 KB + K 3x32 KB + V 3x32 KB = 224 KB, one CTA per SM.
// Every wait is bounded; on a timeout the CTA drains its in-flight copies and
// MMAs, frees its tensor memory and exits with the error word set.
#pragma once

#include "lcsa_device.cuh"

namespace lcsa {

constexpr int K_STAGES = 3;
constexpr int V_STAGES = 3;
constexpr int S_BUFS = 3;
// a K stage is free once the score product that read it has completed, a V
// stage once its PV has: the stages reuse the score buffers' barriers
static_assert(K_STAGES == S_BUFS && V_STAGES == S_BUFS, "K/V stages follow the score buffers");

template <int D>
struct AttnLayout {
  static constexpr int TILE_BYTES = 128 * D * 2;   // 128 tokens x D bf16
  static constexpr int CHUNK_BYTES = 128 * 128;    // 128 rows x 64 channels (one swizzle column)
  static constexpr int BOX_BYTES = 64 * 128;       // one frame of a block, 64 channels
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + K_STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + V_STAGES * TILE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = OFF_BAR + BAR_BYTES + 1024;  // + alignment slack
};

// mbarrier slots
enum : int {
  B_Q_FULL = 0,
  B_K_FULL = 1,                        // K_STAGES
  B_V_FULL = B_K_FULL + K_STAGES,      // V_STAGES
  B_S_FULL = B_V_FULL + V_STAGES,      // S_BUFS; S_j done also frees K stage j % K_STAGES
  B_P_FULL = B_S_FULL + S_BUFS,        // S_BUFS (128 softmax arrivals)
  B_PV_DONE = B_P_FULL + S_BUFS,       // S_BUFS; PV_j done also frees V stage j % V_STAGES
  B_DRAIN = B_PV_DONE + S_BUFS,
  B_COUNT = B_DRAIN + 1
};

constexpr int ATTN_THREADS = 224;
constexpr int SOFTMAX_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O_COL = 128 * S_BUFS;

struct AttnParams {
  const int32_t* blk_idx;    // [B*H][nQB][kmax]
  const int32_t* blk_cnt;    // [B*H][nQB]
  __nv_bfloat16* o;
  float* lse;                // [B*H][Tq][Y][X] or null
  int64_t osh, ost, osy, osx;  // strides of o (stream stride = H * osh)
  int32_t H, Tq, Y, X, Hb, Wb, nQT, nQB, kmax, cap;
  int32_t win, win_mode;     // token-level window (0: none), mode 2 truncate / 3 preserve
  int32_t split_from;        // units >= split_from run as two CTAs over halves of their kept blocks
  float* part_o;             // [split units][2][128][D] fp32 O of each half (normalised), or null
  float* part_lse;           // [split units][2][128] natural-log LSE of each half
  float scale_log2;          // log2(e) / sqrt(D)
  uint64_t wait_limit_ns;
  unsigned int* err;
  int64_t kv_begin[64];
  int64_t kv_end[64];
};

// Exact n / d and n % d for 0 <= n < 2^22 and d >= 1, from a float
// reciprocal: n and the quotient are below 2^23, so the truncated product is
// within one of the quotient and one correction step makes it exact (checked
// for every n < 2^22 on about a thousand divisors).
struct SmallDiv {
  int d;
  float inv;
  __device__ explicit SmallDiv(int d_) : d(d_), inv(1.0f / static_cast<float>(d_)) {}
  __device__ __forceinline__ void divmod(int n, int& q, int& r) const {
    q = __float2int_rz(__int2float_rn(n) * inv);
    r = n - q * d;
    if (r < 0) {
      --q;
      r += d;
    } else if (r >= d) {
      ++q;
      r -= d;
    }
  }
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

// D[tmem] (+)= A[tmem] * B[smem]^T: A (128 x 16, bf16 pairs per 32-bit column)
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
  // CTA -> work unit. A grid whose last wave would be partly empty runs each of
  // its last units as two CTAs over the two halves of the unit's kept blocks;
  // attn_merge_kernel combines the halves.
  int unit = blockIdx.x, half = -1;
  if (static_cast<int>(blockIdx.x) >= p.split_from) {
    const int k = blockIdx.x - p.split_from;
    unit = p.split_from + (k >> 1);
    half = k & 1;
  }
  const int bh = unit / p.nQB;
  const int rr = unit % p.nQB;
  const int tq = p.nQT - 1 - rr / HbWb;
  const int sp = rr % HbWb;
  const int b = bh / p.H;
  const int yq = sp / p.Wb, xq = sp % p.Wb;
  const int64_t row = static_cast<int64_t>(bh) * p.nQB + tq * HbWb + sp;
  const int32_t* blist = p.blk_idx + row * p.kmax;
  // the first two kept block ids go out with the count instead of after it (a
  // second L2 round trip before the first copies); only the second half of a
  // split unit, whose list starts further on, reloads them
  int pre0 = blist[0];
  int pre1 = p.kmax > 1 ? blist[1] : 0;
  int n = p.blk_cnt[row];
  if (n < 0 || n > p.kmax) {
    if (threadIdx.x == 0) atomicOr(p.err, DEVERR_BOUNDS);
    n = 0;
  }
  if (half >= 0) {
    const int h0 = (n + 1) >> 1;
    if (half == 0) {
      n = h0;
    } else {
      blist += h0;
      n -= h0;
      pre0 = n > 0 ? blist[0] : 0;
      pre1 = n > 1 ? blist[1] : 0;
    }
  }
  const int64_t begin = p.kv_begin[b], end = p.kv_end[b];
  const int64_t m_first = begin >> 1;
  const int nkb = static_cast<int>((end >> 1) - m_first) * HbWb;  // valid block ids
  const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;   // older frame of the query block (-1: missing)

  auto checked = [&](int blk) -> int {
    if (blk < 0 || blk >= nkb) {
      atomicOr(p.err, DEVERR_BOUNDS);
      blk = 0;
    }
    return blk;
  };
  // One 128-token tile = 2 frames x D/64 channel columns of 8 KB boxes.
  auto load_tile = [&](const CUtensorMap* map, uint32_t dst, uint32_t bar_full, int x8, int y8,
                       int fr0, int fr1) {
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_5d(dst + c * L::CHUNK_BYTES, map, bar_full, c * 64, x8, y8, fr0, bh);
      tma_load_5d(dst + c * L::CHUNK_BYTES + L::BOX_BYTES, map, bar_full, c * 64, x8, y8, fr1, bh);
    }
  };
  // Ring slots of a key block's two frames; a one-frame block loads its frame twice.
  // The host passes frame numbers shifted down by whole multiples of the ring
  // capacity, so they lie in [0, 2 cap): a ring slot is one conditional
  // subtract. The divisions use SmallDiv (a few instructions, not a software
  // integer division): the producers share sub-partitions with softmax warps.
  const int cap = p.cap;
  const int begin32 = static_cast<int>(begin), m_first32 = static_cast<int>(m_first);
  const SmallDiv div_blocks(HbWb), div_row(p.Wb);
  auto tile_coords = [&](int blk, int& x8, int& y8, int& s0, int& s1) {
    int tk, spk, yb, xb;
    div_blocks.divmod(blk, tk, spk);
    div_row.divmod(spk, yb, xb);
    const int a1 = 2 * (m_first32 + tk) + 1;
    const int a0 = a1 - 1 < begin32 ? a1 : a1 - 1;
    s0 = a0 >= cap ? a0 - cap : a0;
    s1 = a1 >= cap ? a1 - cap : a1;
    x8 = 8 * xb;
    y8 = 8 * yb;
  };

  if (threadIdx.x == 0) {
    // thread 0 is also the Q/K producer: it initialises the barriers and starts
    // the Q and first K copies right away, so their latency overlaps the
    // tensor-memory allocation and the CTA-wide barrier
    const int first_blk = pre0;
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(bar(i), (i >= B_P_FULL && i < B_P_FULL + S_BUFS) ? SOFTMAX_THREADS : 1u);
    *abort_flag = 0;
    mbar_init_fence();
    if (n > 0) {
      mbar_arrive_expect_tx(bar(B_Q_FULL), L::TILE_BYTES);
      // a missing older query frame is replaced by the newer one (rows not stored)
      load_tile(&tmQ, sbase + L::OFF_Q, bar(B_Q_FULL), 8 * xq, 8 * yq, fq0 < 0 ? fq0 + 1 : fq0, fq0 + 1);
      int x8, y8, s0, s1;
      tile_coords(checked(first_blk), x8, y8, s0, s1);
      mbar_arrive_expect_tx(bar(B_K_FULL), L::TILE_BYTES);
      load_tile(&tmK, sbase + L::OFF_K, bar(B_K_FULL), x8, y8, s0, s1);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx w{p.wait_limit_ns, abort_flag, p.err};

  if (warp == 0) {
    // ------------------------------------------------------------ Q + K producer
    if (lane == 0 && n > 0) {
      int issued_k = 1;                           // Q and K_0 went out before the CTA barrier
      int next_blk = n > 1 ? checked(pre1) : 0;
      for (int j = 1; j < n; ++j) {
        const int blk = next_blk;
        if (j + 1 < n) next_blk = checked(blist[j + 1]);
        int x8, y8, s0, s1;
        tile_coords(blk, x8, y8, s0, s1);
        const int ks = j % K_STAGES;
        if (j >= K_STAGES && !wait_bounded(bar(B_S_FULL + ks), ((j / K_STAGES) - 1) & 1, w)) break;
        mbar_arrive_expect_tx(bar(B_K_FULL + ks), L::TILE_BYTES);
        load_tile(&tmK, sbase + L::OFF_K + ks * L::TILE_BYTES, bar(B_K_FULL + ks), x8, y8, s0, s1);
        issued_k = j + 1;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA goes away
        drain_wait(bar(B_Q_FULL), 0, w.limit_ns);
        for (int j = issued_k > K_STAGES ? issued_k - K_STAGES : 0; j < issued_k; ++j)
          drain_wait(bar(B_K_FULL + j % K_STAGES), (j / K_STAGES) & 1, w.limit_ns);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V producer
    if (lane == 0 && n > 0) {
      int issued_v = 0;
      int next_blk = checked(pre0);
      for (int j = 0; j < n; ++j) {
        const int blk = next_blk;
        if (j + 1 < n) next_blk = checked(blist[j + 1]);
        int x8, y8, s0, s1;
        tile_coords(blk, x8, y8, s0, s1);
        const int vs = j % V_STAGES;
        if (j >= V_STAGES && !wait_bounded(bar(B_PV_DONE + vs), ((j / V_STAGES) - 1) & 1, w)) break;
        mbar_arrive_expect_tx(bar(B_V_FULL + vs), L::TILE_BYTES);
        load_tile(&tmV, sbase + L::OFF_V + vs * L::TILE_BYTES, bar(B_V_FULL + vs), x8, y8, s0, s1);
        issued_v = j + 1;
      }
      if (*abort_flag) {
        for (int j = issued_v > V_STAGES ? issued_v - V_STAGES : 0; j < issued_v; ++j)
          drain_wait(bar(B_V_FULL + j % V_STAGES), (j / V_STAGES) & 1, w.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t ID_PV = idesc_bf16_f32(128, D, true);
      auto issue_s = [&](int j) -> bool {
        const int ks = j % K_STAGES;
        if (!wait_bounded(bar(B_K_FULL + ks), (j / K_STAGES) & 1, w)) return false;
        tc_fence_after();
        // one descriptor per operand; a step's is the base plus its byte offset
        // / 16 (the 14-bit address field: shared addresses stay below 2^18)
        const uint64_t qd = desc_sw128(sbase + L::OFF_Q, 16, 1024);
        const uint64_t kd = desc_sw128(sbase + L::OFF_K + ks * L::TILE_BYTES, 16, 1024);
        const uint32_t sd = tmem + (j % S_BUFS) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // K-major operands: 16 channels = 32 bytes inside a 128-byte swizzled row
          const uint32_t off16 = ((kk >> 2) * L::CHUNK_BYTES + (kk & 3) * 32) >> 4;
          umma_ss(sd, qd + off16, kd + off16, ID_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(B_S_FULL + j % S_BUFS));
        return true;
      };
      bool ok = wait_bounded(bar(B_Q_FULL), 0, w);
      if (ok) {
        tc_fence_after();
        ok = issue_s(0);
        if (ok && n > 1) ok = issue_s(1);
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 2 < n) {
          // S_{j+2} overwrites the buffer PV_{j-1} read P_{j-1} from. MMAs into
          // different accumulators are not ordered, so wait until PV_{j-1} has
          // completed. S_{j+2} goes out ahead of PV_j: it does not need P_j, so
          // the softmax of block j+2 does not wait for the issue of PV_j.
          if (j >= 1 && !(ok = wait_bounded(bar(B_PV_DONE + (j - 1) % S_BUFS), ((j - 1) / S_BUFS) & 1, w))) break;
          if (!(ok = issue_s(j + 2))) break;
        }
        const int sb = j % S_BUFS;
        const int vs = j % V_STAGES;
        if (!(ok = wait_bounded(bar(B_P_FULL + sb), (j / S_BUFS) & 1, w))) break;
        if (!(ok = wait_bounded(bar(B_V_FULL + vs), (j / V_STAGES) & 1, w))) break;
        tc_fence_after();
        const uint32_t va = sbase + L::OFF_V + vs * L::TILE_BYTES;
        const uint64_t vd = desc_sw128(va, L::CHUNK_BYTES, 1024);
        const uint32_t pa = tmem + sb * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = P (16 keys = 8 packed columns of S_j's TMEM buffer); B = V
          // (MN-major: channels contiguous), 16 keys = 16 rows of 128 bytes,
          // 64-channel columns 16 KB apart.
          umma_ts(tmem + TMEM_O_COL, pa + kk * 8, vd + kk * (2048 >> 4), ID_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar(B_PV_DONE + sb));
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
    const uint64_t sc2 = f2_pack(scale, scale);
    float m_run = -INFINITY, l_run = 0.f;         // running max (log2 units) and sum
    bool done = n > 0;
    int next_blk = n > 0 ? checked(pre0) : 0;
    int raw_blk = pre1;
    // token-level window of this row's query token (a key token is visible iff
    // its y and x lie in these ranges)
    int wy0 = 0, wy1 = 0, wx0 = 0, wx1 = 0;
    if (p.win > 0) {
      token_window(8 * yq + ((r >> 3) & 7), p.Y, p.win, p.win_mode, wy0, wy1);
      token_window(8 * xq + (r & 7), p.X, p.win, p.win_mode, wx0, wx1);
    }
    for (int j = 0; j < n; ++j) {
      const int sb = j % S_BUFS;
      const int blk = next_blk;
      const bool partial = oldest_partial && blk < HbWb;
      // block j+1's id was loaded one block ago and block j+2's is loaded now:
      // the load's latency never stalls the row
      if (j + 1 < n) next_blk = checked(raw_blk);
      if (j + 2 < n) raw_blk = blist[j + 2];
      if (!warp_wait(bar(B_S_FULL + sb), (j / S_BUFS) & 1, w)) { done = false; break; }
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
      if (p.win > 0) {
        // rows / columns of the key block (8 x 8 tokens, both frames alike) inside the window
        int tk, spk, yb, xb;
        div_blocks.divmod(blk, tk, spk);
        div_row.divmod(spk, yb, xb);
        const int ry = 8 * yb, rx = 8 * xb;
        const int ylo = min(max(wy0 - ry, 0), 8), yhi = min(max(wy1 - ry, 0), 8);
        const int xlo = min(max(wx0 - rx, 0), 8), xhi = min(max(wx1 - rx, 0), 8);
        const uint32_t ym = ((1u << yhi) - 1u) & ~((1u << ylo) - 1u);
        const uint32_t xm = ((1u << xhi) - 1u) & ~((1u << xlo) - 1u);
        if (ym != 0xFFu || xm != 0xFFu) {
          // 64-bit visibility of the frame's 8 x 8 tokens (bit 8*yy + xx): the
          // x mask in every byte, kept for the rows in the window; the block's
          // two frames share it
          const uint64_t xrep = static_cast<uint64_t>(xm) * 0x0101010101010101ull;
          const uint64_t yhi_m = yhi >= 8 ? ~0ull : (1ull << (8 * yhi)) - 1ull;
          const uint64_t ylo_m = ylo >= 8 ? ~0ull : (1ull << (8 * ylo)) - 1ull;
          const uint64_t vis = xrep & yhi_m & ~ylo_m;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            if (!((vis >> c) & 1ull)) {
              s[c] = __float_as_uint(-INFINITY);
              s[c + 64] = __float_as_uint(-INFINITY);
            }
          }
        }
      }
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; c += 8) {
        a0 = fmax3(a0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
        a1 = fmax3(a1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        a2 = fmax3(a2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
        a3 = fmax3(a3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
      }
      const float mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * scale;  // scale > 0
      float m_new = m_run;
      if (j == 0 || mx > m_run + 8.f) m_new = mx;
      if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
        // O may only be rescaled once PV_{j-1} has finished
        if (!warp_wait(bar(B_PV_DONE + (j - 1) % S_BUFS), ((j - 1) / S_BUFS) & 1, w)) { done = false; break; }
        tc_fence_after();
        // 1 for rows whose max did not change (also rows still at -inf, where the difference is NaN)
        const float alpha = m_new == m_run ? 1.f : ex2_approx(m_run - m_new);
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
      // a row that has seen no visible key yet keeps m = -inf; its exponentials use 0
      const float m_ref = m_run == -INFINITY ? 0.f : m_run;
      const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
      uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1])), sc2, nm2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        const uint64_t e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        if (c & 1) acc1 = f2_add(acc1, e2);
        else acc0 = f2_add(acc0, e2);
        float e0, e1;
        f2_unpack(e2, e0, e1);
        pk[c] = pack_bf16x2_rn(e0, e1);
      }
      {
        float s0, s1, s2, s3;
        f2_unpack(acc0, s0, s1);
        f2_unpack(acc1, s2, s3);
        l_run += (s0 + s1) + (s2 + s3);
      }
      // P_j over the first 64 columns of S_j's buffer (S_j has been read)
      tmem_st_32x32b_x32(t_lane + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st_32x32b_x32(t_lane + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_P_FULL + sb));
    }
    if (done) done = warp_wait(bar(B_PV_DONE + (n - 1) % S_BUFS), ((n - 1) / S_BUFS) & 1, w);
    const bool row_valid = !(fq0 < 0 && r < 64);
    const int f = r >> 6, yy = (r >> 3) & 7, xx = r & 7;
    const int frame = fq0 + f;
    const int y = 8 * yq + yy, x = 8 * xq + xx;
    __nv_bfloat16* orow = p.o + static_cast<int64_t>(bh) * p.osh + static_cast<int64_t>(frame) * p.ost +
                          static_cast<int64_t>(y) * p.osy + static_cast<int64_t>(x) * p.osx;
    if (half >= 0) {
      // one half of a split unit: fp32 O (normalised) and LSE for the merge
      const int64_t prow = (static_cast<int64_t>(unit - p.split_from) * 2 + half) * 128 + r;
      float* po = p.part_o + prow * D;
      if (done) tc_fence_after();
      const float inv_l = done && l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (done) {
          tmem_ld_32x32b_x32(t_lane + TMEM_O_COL + c0, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          *reinterpret_cast<float4*>(po + c0 + k) =
              make_float4(__uint_as_float(o[k]) * inv_l, __uint_as_float(o[k + 1]) * inv_l,
                          __uint_as_float(o[k + 2]) * inv_l, __uint_as_float(o[k + 3]) * inv_l);
      }
      p.part_lse[prow] = done && l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    } else if (done) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;   // a row with no visible key: O = 0
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
            l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
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

// Combines the two halves of each split unit, one warp per query row:
// O = (w0 O0 + w1 O1) / (w0 + w1) with w_h = exp(LSE_h - max), LSE = max + log(w0 + w1).
template <int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const __grid_constant__ AttnParams p, int32_t n_split) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<int64_t>(n_split) * 128) return;
  const int su = static_cast<int>(wid >> 7), r = static_cast<int>(wid & 127);
  const int unit = p.split_from + su;
  const int HbWb = p.Hb * p.Wb;
  const int bh = unit / p.nQB, rr = unit % p.nQB;
  const int tq = p.nQT - 1 - rr / HbWb, sp = rr % HbWb;
  const int fq0 = p.Tq - 2 * p.nQT + 2 * tq;
  if (fq0 < 0 && r < 64) return;                   // rows of a missing older frame
  const int frame = fq0 + (r >> 6);
  const int y = 8 * (sp / p.Wb) + ((r >> 3) & 7), x = 8 * (sp % p.Wb) + (r & 7);
  const int64_t r0 = (static_cast<int64_t>(su) * 2) * 128 + r, r1 = r0 + 128;
  const float l0 = p.part_lse[r0], l1 = p.part_lse[r1];
  const float mx = fmaxf(l0, l1);
  float w0 = 0.f, w1 = 0.f, lse = -INFINITY;
  if (mx != -INFINITY) {
    w0 = __expf(l0 - mx);
    w1 = __expf(l1 - mx);
    const float sum = w0 + w1;
    lse = mx + __logf(sum);
    w0 /= sum;
    w1 /= sum;
  }
  __nv_bfloat16* orow = p.o + static_cast<int64_t>(bh) * p.osh + static_cast<int64_t>(frame) * p.ost +
                        static_cast<int64_t>(y) * p.osy + static_cast<int64_t>(x) * p.osx;
  const float* o0 = p.part_o + r0 * D;
  const float* o1 = p.part_o + r1 * D;
  for (int c = 2 * lane; c < D; c += 64) {
    const float2 a = *reinterpret_cast<const float2*>(o0 + c);
    const float2 b = *reinterpret_cast<const float2*>(o1 + c);
    *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16x2(w0 * a.x + w1 * b.x, w0 * a.y + w1 * b.y);
  }
  if (lane == 0 && p.lse != nullptr)
    p.lse[((static_cast<int64_t>(bh) * p.Tq + frame) * p.Y + y) * p.X + x] = lse;
}

}  // namespace lcsa
