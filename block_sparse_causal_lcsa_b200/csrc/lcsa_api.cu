// Host side of liblcsa.so: the C ABI declared in include/lcsa.h. Validates
// every argument before launching, encodes the TMA tensor maps, sizes the
// grids and launches the sm_100a kernels on the caller's stream. Allocates no
// memory: the device state of the library is its per-device error word and
// the fixed scratch array of lcsa_select_blocks_noalloc.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "lcsa.h"
#include "attn_fwd.cuh"
#include "attn_bwd.cuh"
#include "kv_append.cuh"
#include "ingest.cuh"
#include "segment.cuh"
#include "select.cuh"

// Scratch of lcsa_select_blocks_noalloc: the score keys that the caller's
// workspace holds in lcsa_select_blocks. A module-scope array, so it exists on
// every device that loads this library's kernels, until the process exits.
// In host code the name is only a handle for cudaGetSymbolAddress.
static __device__ __align__(256) uint64_t lcsa_select_scratch[LCSA_SELECT_STATIC_SCRATCH_BYTES / sizeof(uint64_t)];

namespace lcsa {

// Error word shared by all kernels of this library on one device.
__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultWaitNs = 1000000000ull;  // 1 s
uint64_t g_wait_limit_ns = kDefaultWaitNs;

std::mutex g_mu;
unsigned int* g_err_ptr[kMaxDevices] = {};
bool g_attr_done[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Current device, its error-word address and one-time kernel attributes.
lcsa_status device_setup(int* dev_out, unsigned int** err_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LCSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_device_error) != cudaSuccess) return LCSA_ERR_CUDA;
    g_err_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  if (!g_attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnLayout<128>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnLayout<64>::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(score_smem_bytes(128))) != cudaSuccess ||
        cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(score_smem_bytes(64))) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdLayout<128>::SMEM_DQ) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdLayout<64>::SMEM_DQ) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dkdv_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdLayout<128>::SMEM_KV) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dkdv_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             BwdLayout<64>::SMEM_KV) != cudaSuccess)
      return LCSA_ERR_CUDA;
    if (cudaDeviceGetAttribute(&g_sm_count[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        g_sm_count[dev] < 1)
      return LCSA_ERR_CUDA;
    g_attr_done[dev] = true;
  }
  if (g_encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return LCSA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *dev_out = dev;
  *err_out = g_err_ptr[dev];
  return LCSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Checks common to every token tensor.
lcsa_status check_tensor(const lcsa_tensor* t) {
  if (t == nullptr || t->data == nullptr) return LCSA_ERR_INVALID_ARG;
  if (t->B < 1 || t->H < 1 || t->T < 1 || t->Y < 8 || t->X < 8) return LCSA_ERR_SHAPE;
  if (t->D != 64 && t->D != 128) return LCSA_ERR_SHAPE;
  if (t->Y % 8 || t->X % 8) return LCSA_ERR_SHAPE;
  if (t->B > LCSA_MAX_STREAMS) return LCSA_ERR_SHAPE;
  if (!aligned16(t->data)) return LCSA_ERR_ALIGN;
  const int64_t s[5] = {t->stride_b, t->stride_h, t->stride_t, t->stride_y, t->stride_x};
  for (int i = 0; i < 5; ++i)
    if (s[i] <= 0 || s[i] % 8) return LCSA_ERR_ALIGN;
  if (t->stride_b != static_cast<int64_t>(t->H) * t->stride_h) return LCSA_ERR_SHAPE;
  if (t->stride_x < t->D) return LCSA_ERR_SHAPE;
  return LCSA_OK;
}

lcsa_status check_cache(const lcsa_kv_cache* kv) {
  if (kv == nullptr || kv->k == nullptr || kv->v == nullptr || kv->k_pool == nullptr)
    return LCSA_ERR_INVALID_ARG;
  if (kv->B < 1 || kv->B > LCSA_MAX_STREAMS || kv->H < 1) return LCSA_ERR_SHAPE;
  if (kv->D != 64 && kv->D != 128) return LCSA_ERR_SHAPE;
  if (kv->Y < 8 || kv->X < 8 || kv->Y % 8 || kv->X % 8) return LCSA_ERR_SHAPE;
  if (kv->cap_frames < 2 || kv->cap_frames % 2) return LCSA_ERR_SHAPE;
  if (!aligned16(kv->k) || !aligned16(kv->v) || !aligned16(kv->k_pool)) return LCSA_ERR_ALIGN;
  for (int b = 0; b < kv->B; ++b) {
    const int64_t n = kv->end[b] - kv->begin[b];
    if (kv->begin[b] < 0 || n < 0 || n > kv->cap_frames || (kv->end[b] & 1)) return LCSA_ERR_INVALID_ARG;
  }
  return LCSA_OK;
}

int temporal_blocks(int frames) { return (frames + 1) / 2; }

// 5-D map (d, x, y, frame, stream*head) over bf16 tokens; box = 64 channels x
// 8 x 8 tokens x 1 frame, 128-byte swizzle.
lcsa_status encode_map(CUtensorMap* map, void* data, int B, int H, int T, int Y, int X, int D,
                       int64_t sh, int64_t st, int64_t sy, int64_t sx) {
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(X),
                              static_cast<cuuint64_t>(Y), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(B) * H};
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(sx) * 2, static_cast<cuuint64_t>(sy) * 2,
                                 static_cast<cuuint64_t>(st) * 2, static_cast<cuuint64_t>(sh) * 2};
  const cuuint32_t box[5] = {64, 8, 8, 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, data, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LCSA_OK : LCSA_ERR_CUDA;
}

// One thread waits on a barrier that nothing arrives at: the bounded wait
// must give up, set the error word and return (test of the timeout path).
__global__ void stalled_wait_kernel(uint64_t limit_ns, unsigned int* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    mbar_init_fence();
    const WaitCtx w{limit_ns, &abort_flag, err};
    wait_bounded(smem_u32(&bar), 0, w);
  }
}

// Evaluates the FMA-pipe 2^x polynomial (exp2_poly_f2) elementwise.
__global__ void exp2_poly_kernel(const float* x, float* y, int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    float a, b;
    f2_unpack(exp2_poly_f2(f2_pack(x[i], x[i + 1])), a, b);
    y[i] = a;
    y[i + 1] = b;
  } else if (i < n) {
    float a, b;
    f2_unpack(exp2_poly_f2(f2_pack(x[i], 0.f)), a, b);
    y[i] = a;
  }
}

lcsa_status launched() { return cudaGetLastError() == cudaSuccess ? LCSA_OK : LCSA_ERR_CUDA; }

// K_i upper bound over the rows of a selection (largest C_i gives largest K_i).
int32_t kmax_for(int nKT, int nQT, int Hb, int Wb, const lcsa_select_params* p) {
  if (nKT < nQT || nQT < 1) return 0;
  int wy = Hb, wx = Wb;
  if (p->window > 0) {
    // widest window over all query blocks along each axis
    wy = 0;
    wx = 0;
    for (int i = 0; i < Hb; ++i) {
      int lo, hi;
      window_bounds(i, Hb, p->window, p->window_mode, lo, hi);
      wy = hi - lo > wy ? hi - lo : wy;
    }
    for (int i = 0; i < Wb; ++i) {
      int lo, hi;
      window_bounds(i, Wb, p->window, p->window_mode, lo, hi);
      wx = hi - lo > wx ? hi - lo : wx;
    }
  }
  const int C = nKT * wy * wx;
  if (p->top_k > 0) return p->top_k < C ? p->top_k : C;
  int K = static_cast<int>(std::ceil(p->density * static_cast<double>(C)));
  if (K < 1) K = 1;
  return K < C ? K : C;
}

void set_ingest_source(IngestTensor& it, const lcsa_tensor* t) {
  it.src = static_cast<const __nv_bfloat16*>(t->data);
  it.sb = t->stride_b; it.sh = t->stride_h; it.st = t->stride_t;
  it.sy = t->stride_y; it.sx = t->stride_x;
  it.T = t->T;
  it.nT = temporal_blocks(t->T);
}

// One CTA per block of every tensor of p (a tensor with 0 units is skipped).
lcsa_status launch_ingest(const IngestParams& p, int D, cudaStream_t cs) {
  const int64_t grid = p.t[0].units + p.t[1].units + p.t[2].units;
  if (grid > 0x7fffffff) return LCSA_ERR_SHAPE;
  if (grid == 0) return LCSA_OK;
  if (D == 128) ingest_kernel<128><<<static_cast<unsigned>(grid), INGEST_THREADS, 0, cs>>>(p);
  else ingest_kernel<64><<<static_cast<unsigned>(grid), INGEST_THREADS, 0, cs>>>(p);
  return launched();
}

// Frame numbers as the kernels see them: shifted down by whole multiples of the
// ring capacity. Ring slots (a % cap, m % (cap/2) with cap even), the parity of
// begin and all lengths are unchanged, so the launches of a steady stream
// repeat with the period of the ring and can be replayed from a CUDA graph.
int64_t ring_base(int64_t begin, int cap) { return begin >= 0 ? begin - begin % cap : 0; }

// Cache state after appending Tn frames to streams [offset, offset+n): the
// absolute frame of the chunk's first frame, and the new begin / end.
lcsa_status append_state(const lcsa_kv_cache* kv, int Tn, int n, int offset, int64_t* first, int64_t* nb,
                         int64_t* ne) {
  for (int bn = 0; bn < n; ++bn) {
    const int b = bn + offset;
    const bool empty = kv->end[b] == kv->begin[b];
    if (!empty && (Tn & 1)) return LCSA_ERR_SHAPE;  // odd chunks only start a stream
    first[bn] = empty ? kv->end[b] + (Tn & 1) : kv->end[b];
    const int64_t e = first[bn] + Tn;
    const int64_t old_begin = empty ? first[bn] : kv->begin[b];
    ne[bn] = e;
    nb[bn] = old_begin > e - kv->cap_frames ? old_begin : e - kv->cap_frames;
  }
  return LCSA_OK;
}

}  // namespace
}  // namespace lcsa

using namespace lcsa;

extern "C" {

int32_t lcsa_abi_version(void) { return LCSA_ABI_VERSION; }

const char* lcsa_status_string(lcsa_status s) {
  switch (s) {
    case LCSA_OK: return "ok";
    case LCSA_ERR_INVALID_ARG: return "invalid argument";
    case LCSA_ERR_SHAPE: return "unsupported or inconsistent shape";
    case LCSA_ERR_ALIGN: return "misaligned pointer or stride";
    case LCSA_ERR_CAPACITY: return "capacity exceeded";
    case LCSA_ERR_WORKSPACE: return "workspace error";
    case LCSA_ERR_CUDA: return "CUDA error";
    case LCSA_ERR_TIMEOUT: return "a kernel wait timed out";
    case LCSA_ERR_DEVICE_BOUNDS: return "a kernel saw an out-of-range block id";
    case LCSA_ERR_SCRATCH_LIMIT: return "request exceeds the library's fixed scratch array";
  }
  return "unknown status";
}

lcsa_status lcsa_pool_qk(const lcsa_tensor* q, const lcsa_tensor* k, double* q_pool, double* k_pool,
                         lcsa_stream_t stream) {
  lcsa_status s = check_tensor(q);
  if (s != LCSA_OK) return s;
  if (q_pool == nullptr || !aligned16(q_pool)) return q_pool ? LCSA_ERR_ALIGN : LCSA_ERR_INVALID_ARG;
  if (k != nullptr) {
    if ((s = check_tensor(k)) != LCSA_OK) return s;
    if (k->B != q->B || k->H != q->H || k->Y != q->Y || k->X != q->X || k->D != q->D) return LCSA_ERR_SHAPE;
    if (k_pool == nullptr || !aligned16(k_pool)) return k_pool ? LCSA_ERR_ALIGN : LCSA_ERR_INVALID_ARG;
  }
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  IngestParams p{};
  p.H = q->H; p.Y = q->Y; p.X = q->X;
  p.Hb = q->Y / 8;
  p.Wb = q->X / 8;
  p.cap = 2;  // no ring destination
  const lcsa_tensor* ts[2] = {q, k};
  double* outs[2] = {q_pool, k_pool};
  for (int i = 0; i < 2; ++i) {
    IngestTensor& it = p.t[i];
    if (ts[i] == nullptr) continue;  // units 0
    set_ingest_source(it, ts[i]);
    it.tb_first = 0;
    it.units = static_cast<int64_t>(ts[i]->B) * ts[i]->H * it.nT * p.Hb * p.Wb;
    it.pool_out = outs[i];
  }
  return launch_ingest(p, q->D, static_cast<cudaStream_t>(stream));
}

// lcsa_kv_append, optionally with the pooling of q into q_pool in the same
// launch (only on the fused path, where K is pooled while it is copied).
static lcsa_status kv_append_impl(lcsa_kv_cache* kv, const lcsa_tensor* k_new, const lcsa_tensor* v_new,
                                  const double* k_pool_new, int32_t stream_offset, lcsa_stream_t stream,
                                  const lcsa_tensor* q, double* q_pool) {
  lcsa_status s = check_cache(kv);
  if (s != LCSA_OK) return s;
  if ((s = check_tensor(k_new)) != LCSA_OK || (s = check_tensor(v_new)) != LCSA_OK) return s;
  if (k_pool_new != nullptr && !aligned16(k_pool_new)) return LCSA_ERR_ALIGN;
  const lcsa_tensor* kn = k_new;
  if (v_new->B != kn->B || v_new->H != kn->H || v_new->T != kn->T || v_new->Y != kn->Y ||
      v_new->X != kn->X || v_new->D != kn->D)
    return LCSA_ERR_SHAPE;
  if (kn->H != kv->H || kn->Y != kv->Y || kn->X != kv->X || kn->D != kv->D) return LCSA_ERR_SHAPE;
  if (stream_offset < 0 || stream_offset + kn->B > kv->B) return LCSA_ERR_INVALID_ARG;
  const int Tn = kn->T;
  const int cap = kv->cap_frames;
  AppendParams p{};
  int64_t new_begin[LCSA_MAX_STREAMS], new_end[LCSA_MAX_STREAMS], first[LCSA_MAX_STREAMS];
  if ((s = append_state(kv, Tn, kn->B, stream_offset, first, new_begin, new_end)) != LCSA_OK) return s;
  for (int bn = 0; bn < kn->B; ++bn) p.first_abs[bn] = first[bn] - ring_base(first[bn], cap);
  // Every stream of one call appends the same frames of the chunk: the newest
  // min(Tn, cap) frames (cap is even, so the kept blocks are whole or the
  // chunk's own one-frame oldest block).
  const int f_first = Tn > cap ? Tn - cap : 0;
  const int nTn = temporal_blocks(Tn);
  const int copy_blocks = temporal_blocks(Tn - f_first);
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  if (k_pool_new == nullptr) {
    // pool K while copying it: one read of K and V, one CTA per block
    IngestParams ip{};
    ip.H = kn->H; ip.Y = kn->Y; ip.X = kn->X;
    ip.Hb = kn->Y / 8; ip.Wb = kn->X / 8;
    ip.cap = cap;
    ip.stream_offset = stream_offset;
    for (int bn = 0; bn < kn->B; ++bn) ip.first_abs[bn] = p.first_abs[bn];
    const lcsa_tensor* ts[2] = {kn, v_new};
    __nv_bfloat16* dsts[2] = {static_cast<__nv_bfloat16*>(kv->k), static_cast<__nv_bfloat16*>(kv->v)};
    for (int i = 0; i < 2; ++i) {
      IngestTensor& it = ip.t[i];
      set_ingest_source(it, ts[i]);
      it.tb_first = nTn - copy_blocks;
      it.units = static_cast<int64_t>(kn->B) * kn->H * copy_blocks * ip.Hb * ip.Wb;
      it.copy_dst = dsts[i];
    }
    ip.t[0].pool_out = kv->k_pool;
    ip.t[0].pool_ring = 1;
    if (q != nullptr) {
      IngestTensor& it = ip.t[2];
      set_ingest_source(it, q);
      it.tb_first = 0;
      it.units = static_cast<int64_t>(q->B) * q->H * it.nT * ip.Hb * ip.Wb;
      it.pool_out = q_pool;
    }
    if ((s = launch_ingest(ip, kn->D, static_cast<cudaStream_t>(stream))) != LCSA_OK) return s;
    for (int bn = 0; bn < kn->B; ++bn) {
      kv->begin[bn + stream_offset] = new_begin[bn];
      kv->end[bn + stream_offset] = new_end[bn];
    }
    return LCSA_OK;
  }
  p.k_new = static_cast<const __nv_bfloat16*>(kn->data);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new->data);
  p.kp_new = k_pool_new;
  p.k_cache = static_cast<__nv_bfloat16*>(kv->k);
  p.v_cache = static_cast<__nv_bfloat16*>(kv->v);
  p.kp_cache = kv->k_pool;
  p.ksb = kn->stride_b; p.ksh = kn->stride_h; p.kst = kn->stride_t; p.ksy = kn->stride_y; p.ksx = kn->stride_x;
  p.vsb = v_new->stride_b; p.vsh = v_new->stride_h; p.vst = v_new->stride_t;
  p.vsy = v_new->stride_y; p.vsx = v_new->stride_x;
  p.Bn = kn->B; p.H = kn->H; p.Y = kn->Y; p.X = kn->X; p.D = kn->D;
  p.Hb = kn->Y / 8; p.Wb = kn->X / 8;
  p.cap = cap;
  p.stream_offset = stream_offset;
  p.f_first = f_first;
  p.n_frames = Tn - f_first;
  p.nTn = nTn;
  p.tb_first = nTn - copy_blocks;
  p.kv_planes = kn->B * kn->H * p.n_frames;
  p.pool_planes = kn->B * kn->H * copy_blocks;
  const int64_t planes = 2 * static_cast<int64_t>(p.kv_planes) + p.pool_planes;
  if (planes > 65535) return LCSA_ERR_SHAPE;
  const int64_t plane_vecs = static_cast<int64_t>(p.Y) * p.X * p.D / 8;
  const int64_t gx = (plane_vecs + APPEND_CHUNK - 1) / APPEND_CHUNK;
  kv_append_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(planes)), APPEND_THREADS, 0,
                     static_cast<cudaStream_t>(stream)>>>(p);
  if ((s = launched()) != LCSA_OK) return s;
  for (int bn = 0; bn < kn->B; ++bn) {
    kv->begin[bn + stream_offset] = new_begin[bn];
    kv->end[bn + stream_offset] = new_end[bn];
  }
  return LCSA_OK;
}

lcsa_status lcsa_kv_append(lcsa_kv_cache* kv, const lcsa_tensor* k_new, const lcsa_tensor* v_new,
                           const double* k_pool_new, int32_t stream_offset, lcsa_stream_t stream) {
  return kv_append_impl(kv, k_new, v_new, k_pool_new, stream_offset, stream, nullptr, nullptr);
}

lcsa_status lcsa_ingest_chunk(const lcsa_tensor* q, double* q_pool, lcsa_kv_cache* kv, const lcsa_tensor* k_new,
                              const lcsa_tensor* v_new, int32_t stream_offset, lcsa_stream_t stream) {
  lcsa_status s = check_tensor(q);
  if (s != LCSA_OK) return s;
  if (kv == nullptr) return LCSA_ERR_INVALID_ARG;
  if (q_pool == nullptr) return LCSA_ERR_INVALID_ARG;
  if (!aligned16(q_pool)) return LCSA_ERR_ALIGN;
  if (q->H != kv->H || q->Y != kv->Y || q->X != kv->X || q->D != kv->D) return LCSA_ERR_SHAPE;
  return kv_append_impl(kv, k_new, v_new, nullptr, stream_offset, stream, q, q_pool);
}

lcsa_status lcsa_kv_advance(lcsa_kv_cache* kv, int32_t frames, int32_t n_streams, int32_t stream_offset) {
  lcsa_status s = check_cache(kv);
  if (s != LCSA_OK) return s;
  if (frames < 1 || n_streams < 1 || stream_offset < 0 || stream_offset + n_streams > kv->B)
    return LCSA_ERR_INVALID_ARG;
  int64_t first[LCSA_MAX_STREAMS], nb[LCSA_MAX_STREAMS], ne[LCSA_MAX_STREAMS];
  if ((s = append_state(kv, frames, n_streams, stream_offset, first, nb, ne)) != LCSA_OK) return s;
  for (int bn = 0; bn < n_streams; ++bn) {
    kv->begin[bn + stream_offset] = nb[bn];
    kv->end[bn + stream_offset] = ne[bn];
  }
  return LCSA_OK;
}

int32_t lcsa_select_kmax(const lcsa_kv_cache* kv, int32_t q_frames, const lcsa_select_params* p) {
  if (kv == nullptr || p == nullptr || q_frames < 1 || kv->B < 1 || kv->B > LCSA_MAX_STREAMS) return 0;
  int nKT = 0;
  for (int b = 0; b < kv->B; ++b) {
    const int n = static_cast<int>((kv->end[b] >> 1) - (kv->begin[b] >> 1));
    nKT = n > nKT ? n : nKT;
  }
  return kmax_for(nKT, temporal_blocks(q_frames), kv->Y / 8, kv->X / 8, p);
}

// Largest number of causal candidates of any query block: the cache's longest
// stream, all of its temporal blocks.
static int64_t select_c_stride(const lcsa_kv_cache* kv) {
  int nKT = 0;
  for (int b = 0; b < kv->B; ++b) {
    const int n = static_cast<int>((kv->end[b] >> 1) - (kv->begin[b] >> 1));
    nKT = n > nKT ? n : nKT;
  }
  return static_cast<int64_t>(nKT) * (kv->Y / 8) * (kv->X / 8);
}

size_t lcsa_select_workspace_bytes(const lcsa_kv_cache* kv, int32_t q_frames) {
  if (kv == nullptr || q_frames < 1 || kv->B < 1 || kv->B > LCSA_MAX_STREAMS || kv->Y < 8 || kv->X < 8)
    return 0;
  const int64_t rows = static_cast<int64_t>(kv->B) * kv->H * temporal_blocks(q_frames) * (kv->Y / 8) * (kv->X / 8);
  return static_cast<size_t>(rows * select_c_stride(kv)) * sizeof(uint64_t);
}

lcsa_status lcsa_select_blocks(const double* q_pool, int32_t q_frames, const lcsa_kv_cache* kv,
                               const lcsa_select_params* sp, int32_t* blk_idx, int32_t* blk_cnt,
                               void* workspace, size_t workspace_bytes, lcsa_stream_t stream) {
  lcsa_status s = check_cache(kv);
  if (s != LCSA_OK) return s;
  if (q_pool == nullptr || sp == nullptr || blk_idx == nullptr || blk_cnt == nullptr || workspace == nullptr)
    return LCSA_ERR_INVALID_ARG;
  if (!aligned16(q_pool) || !aligned16(workspace)) return LCSA_ERR_ALIGN;
  if (sp->top_k < 0 || sp->kmax < 1 || !(sp->tie_eps >= 0.0)) return LCSA_ERR_INVALID_ARG;
  if (sp->top_k == 0 && !(sp->density > 0.0 && sp->density <= 1.0)) return LCSA_ERR_INVALID_ARG;
  if (sp->window_mode < LCSA_WINDOW_TRUNCATE || sp->window_mode > LCSA_WINDOW_PRESERVE_TOKENS)
    return LCSA_ERR_INVALID_ARG;
  // block windows are centred: an odd number of blocks; token windows any width
  if (sp->window < 0 || (sp->window > 0 && sp->window % 2 == 0 && sp->window_mode <= LCSA_WINDOW_PRESERVE))
    return LCSA_ERR_INVALID_ARG;
  if (q_frames < 1) return LCSA_ERR_SHAPE;
  const int Hb = kv->Y / 8, Wb = kv->X / 8, HbWb = Hb * Wb;
  const int nQT = temporal_blocks(q_frames);
  int nKT_max = 0;
  for (int b = 0; b < kv->B; ++b) {
    if (kv->end[b] - kv->begin[b] < q_frames) return LCSA_ERR_SHAPE;  // queries are cached frames
    const int n = static_cast<int>((kv->end[b] >> 1) - (kv->begin[b] >> 1));
    nKT_max = n > nKT_max ? n : nKT_max;
  }
  if (kmax_for(nKT_max, nQT, Hb, Wb, sp) > sp->kmax) return LCSA_ERR_CAPACITY;
  if (workspace_bytes < lcsa_select_workspace_bytes(kv, q_frames)) return LCSA_ERR_WORKSPACE;
  const int64_t c_stride = select_c_stride(kv);
  const int64_t rows = static_cast<int64_t>(kv->B) * kv->H * nQT * HbWb;
  if (c_stride > 2048 || (c_stride + SC_CANDS - 1) / SC_CANDS > 0x7fffffff ||
      static_cast<int64_t>(kv->B) * kv->H * nQT > 65535 || rows > 0x7fffffff)
    return LCSA_ERR_SHAPE;
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  SelectParams p{};
  p.q_pool = q_pool;
  p.k_pool = kv->k_pool;
  p.keys = static_cast<uint64_t*>(workspace);
  p.blk_idx = blk_idx;
  p.blk_cnt = blk_cnt;
  p.B = kv->B; p.H = kv->H; p.Hb = Hb; p.Wb = Wb; p.nQT = nQT;
  p.cap_blk = kv->cap_frames / 2;
  p.top_k = sp->top_k; p.window = sp->window; p.window_mode = sp->window_mode; p.kmax = sp->kmax;
  p.c_stride = static_cast<int32_t>(c_stride);
  p.density = sp->density;
  p.tie_eps = sp->tie_eps;
  p.sqrt_d = std::sqrt(static_cast<double>(kv->D));
  p.err = err;
  for (int b = 0; b < kv->B; ++b) {
    const int64_t base = ring_base(kv->begin[b], kv->cap_frames);
    p.kv_begin[b] = kv->begin[b] - base;
    p.kv_end[b] = kv->end[b] - base;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const dim3 sgrid(static_cast<unsigned>((c_stride + SC_CANDS - 1) / SC_CANDS),
                   static_cast<unsigned>((HbWb + SC_ROWS - 1) / SC_ROWS),
                   static_cast<unsigned>(kv->B * kv->H * nQT));
  if (kv->D == 128) score_kernel<128><<<sgrid, SC_THREADS, score_smem_bytes(128), cs>>>(p);
  else score_kernel<64><<<sgrid, SC_THREADS, score_smem_bytes(64), cs>>>(p);
  if ((s = launched()) != LCSA_OK) return s;
  // a warp per query block, the row's keys in its registers
  const unsigned wgrid = static_cast<unsigned>((rows + TKW_WARPS - 1) / TKW_WARPS);
  if (c_stride <= 256) topk_warp_kernel<8><<<wgrid, TKW_WARPS * 32, 0, cs>>>(p);
  else if (c_stride <= 512) topk_warp_kernel<16><<<wgrid, TKW_WARPS * 32, 0, cs>>>(p);
  else if (c_stride <= 1024) topk_warp_kernel<32><<<wgrid, TKW_WARPS * 32, 0, cs>>>(p);
  else topk_warp_kernel<64><<<wgrid, TKW_WARPS * 32, 0, cs>>>(p);
  return launched();
}

int32_t lcsa_segment_kmax(const lcsa_kv_cache* kv) {
  if (kv == nullptr || kv->B < 1 || kv->B > LCSA_MAX_STREAMS || kv->Y < 8 || kv->X < 8) return 0;
  int nKT = 0;
  for (int b = 0; b < kv->B; ++b) {
    const int n = static_cast<int>((kv->end[b] >> 1) - (kv->begin[b] >> 1));
    nKT = n > nKT ? n : nKT;
  }
  return nKT * (kv->Y / 8) * (kv->X / 8);
}

lcsa_status lcsa_segment_blocks(int32_t q_frames, const lcsa_kv_cache* kv, int32_t kmax, int32_t* blk_idx,
                                int32_t* blk_cnt, lcsa_stream_t stream) {
  lcsa_status s = check_cache(kv);
  if (s != LCSA_OK) return s;
  if (blk_idx == nullptr || blk_cnt == nullptr) return LCSA_ERR_INVALID_ARG;
  if (q_frames < 1) return LCSA_ERR_SHAPE;
  for (int b = 0; b < kv->B; ++b)
    if (kv->end[b] - kv->begin[b] < 1 || kv->end[b] - kv->begin[b] > q_frames) return LCSA_ERR_SHAPE;
  if (kmax < lcsa_segment_kmax(kv)) return LCSA_ERR_CAPACITY;
  const int64_t rows = static_cast<int64_t>(kv->B) * kv->H * temporal_blocks(q_frames) * (kv->Y / 8) * (kv->X / 8);
  if (rows * 32 > 0x7fffffff) return LCSA_ERR_SHAPE;
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  SegmentParams p{};
  p.blk_idx = blk_idx;
  p.blk_cnt = blk_cnt;
  p.H = kv->H;
  p.Tq = q_frames;
  p.nQT = temporal_blocks(q_frames);
  p.HbWb = (kv->Y / 8) * (kv->X / 8);
  p.kmax = kmax;
  p.rows = rows;
  for (int b = 0; b < kv->B; ++b) {
    const int64_t base = ring_base(kv->begin[b], kv->cap_frames);
    p.kv_begin[b] = kv->begin[b] - base;
    p.kv_end[b] = kv->end[b] - base;
  }
  // one warp per query-block row, rows numbered bh * nQB + qb
  segment_blocks_kernel<<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0,
                          static_cast<cudaStream_t>(stream)>>>(p);
  return launched();
}

// Backward workspace: LSE*log2(e) and delta per query row in block order,
// then the per-key-block count and list of the query blocks that kept it.
struct BwdSizes {
  int64_t BH, nQB, nKBmax, off_delta, off_cnt, off_list, total;
};
static BwdSizes bwd_sizes(const lcsa_kv_cache* kv, int32_t q_frames) {
  BwdSizes z{};
  const int64_t HbWb = static_cast<int64_t>(kv->Y / 8) * (kv->X / 8);
  int nKT = 0;
  for (int b = 0; b < kv->B; ++b) {
    const int n = static_cast<int>((kv->end[b] >> 1) - (kv->begin[b] >> 1));
    nKT = n > nKT ? n : nKT;
  }
  z.BH = static_cast<int64_t>(kv->B) * kv->H;
  z.nQB = temporal_blocks(q_frames) * HbWb;
  z.nKBmax = nKT * HbWb;
  const int64_t vec = z.BH * z.nQB * 128 * 4;
  z.off_delta = vec;
  z.off_cnt = 2 * vec;
  z.off_list = z.off_cnt + (z.BH * z.nKBmax * 4 + 15) / 16 * 16;
  z.total = z.off_list + z.BH * z.nKBmax * z.nQB * 4;
  return z;
}

size_t lcsa_sparse_attn_bwd_workspace_bytes(const lcsa_kv_cache* kv, int32_t q_frames) {
  if (kv == nullptr || q_frames < 1 || kv->B < 1 || kv->B > LCSA_MAX_STREAMS || kv->Y < 8 || kv->X < 8)
    return 0;
  return static_cast<size_t>(bwd_sizes(kv, q_frames).total);
}

lcsa_status lcsa_sparse_attn_bwd(const lcsa_tensor* q, const lcsa_kv_cache* kv, const int32_t* blk_idx,
                                 const int32_t* blk_cnt, int32_t kmax, const lcsa_tensor* o, const float* lse,
                                 const lcsa_tensor* d_o, lcsa_tensor* dq, void* dk, void* dv, void* workspace,
                                 size_t workspace_bytes, lcsa_stream_t stream) {
  lcsa_status s = check_tensor(q);
  if (s != LCSA_OK) return s;
  if ((s = check_cache(kv)) != LCSA_OK) return s;
  if (o == nullptr || d_o == nullptr || dq == nullptr) return LCSA_ERR_INVALID_ARG;
  if ((s = check_tensor(o)) != LCSA_OK || (s = check_tensor(d_o)) != LCSA_OK || (s = check_tensor(dq)) != LCSA_OK)
    return s;
  if (blk_idx == nullptr || blk_cnt == nullptr || kmax < 1 || lse == nullptr || dk == nullptr || dv == nullptr ||
      workspace == nullptr)
    return LCSA_ERR_INVALID_ARG;
  if (q->B != kv->B || q->H != kv->H || q->Y != kv->Y || q->X != kv->X || q->D != kv->D) return LCSA_ERR_SHAPE;
  const lcsa_tensor* like_q[3] = {o, d_o, dq};
  for (const lcsa_tensor* t : like_q)
    if (t->B != q->B || t->H != q->H || t->T != q->T || t->Y != q->Y || t->X != q->X || t->D != q->D)
      return LCSA_ERR_SHAPE;
  for (int b = 0; b < kv->B; ++b)
    if (kv->end[b] - kv->begin[b] < 1) return LCSA_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return LCSA_ERR_ALIGN;
  const BwdSizes z = bwd_sizes(kv, q->T);
  if (workspace_bytes < static_cast<size_t>(z.total)) return LCSA_ERR_WORKSPACE;
  if (z.BH * z.nQB > 0x7fffffff || z.BH * z.nKBmax * 32 > 0x7fffffff) return LCSA_ERR_SHAPE;
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  CUtensorMap tq, tdo, tk, tv;
  const int64_t cs_x = kv->D, cs_y = static_cast<int64_t>(kv->X) * kv->D;
  const int64_t cs_t = cs_y * kv->Y, cs_h = cs_t * kv->cap_frames;
  if ((s = encode_map(&tq, q->data, q->B, q->H, q->T, q->Y, q->X, q->D, q->stride_h, q->stride_t, q->stride_y,
                      q->stride_x)) != LCSA_OK ||
      (s = encode_map(&tdo, d_o->data, q->B, q->H, q->T, q->Y, q->X, q->D, d_o->stride_h, d_o->stride_t,
                      d_o->stride_y, d_o->stride_x)) != LCSA_OK ||
      (s = encode_map(&tk, kv->k, kv->B, kv->H, kv->cap_frames, kv->Y, kv->X, kv->D, cs_h, cs_t, cs_y, cs_x)) !=
          LCSA_OK ||
      (s = encode_map(&tv, kv->v, kv->B, kv->H, kv->cap_frames, kv->Y, kv->X, kv->D, cs_h, cs_t, cs_y, cs_x)) !=
          LCSA_OK)
    return s;
  BwdParams p{};
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.blk_idx = blk_idx;
  p.blk_cnt = blk_cnt;
  p.o = static_cast<const __nv_bfloat16*>(o->data);
  p.d_o = static_cast<const __nv_bfloat16*>(d_o->data);
  p.lse = lse;
  p.dq = static_cast<__nv_bfloat16*>(dq->data);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.lse2_blk = reinterpret_cast<float*>(ws);
  p.delta_blk = reinterpret_cast<float*>(ws + z.off_delta);
  p.qcnt = reinterpret_cast<int32_t*>(ws + z.off_cnt);
  p.qlist = reinterpret_cast<int32_t*>(ws + z.off_list);
  p.osh = o->stride_h; p.ost = o->stride_t; p.osy = o->stride_y; p.osx = o->stride_x;
  p.gsh = d_o->stride_h; p.gst = d_o->stride_t; p.gsy = d_o->stride_y; p.gsx = d_o->stride_x;
  p.qsh = dq->stride_h; p.qst = dq->stride_t; p.qsy = dq->stride_y; p.qsx = dq->stride_x;
  p.BH = static_cast<int32_t>(z.BH);
  p.H = q->H; p.Tq = q->T; p.Y = q->Y; p.X = q->X; p.Hb = q->Y / 8; p.Wb = q->X / 8;
  p.nQT = temporal_blocks(q->T);
  p.nQB = static_cast<int32_t>(z.nQB);
  p.kmax = kmax;
  p.cap = kv->cap_frames;
  p.nKBmax = static_cast<int32_t>(z.nKBmax);
  p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(q->D)));
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.wait_limit_ns = g_wait_limit_ns;
  p.err = err;
  for (int b = 0; b < kv->B; ++b) {
    const int64_t base = ring_base(kv->begin[b], kv->cap_frames);
    p.kv_begin[b] = kv->begin[b] - base;
    p.kv_end[b] = kv->end[b] - base;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const unsigned n_q = static_cast<unsigned>(z.BH * z.nQB), n_k = static_cast<unsigned>(z.BH * z.nKBmax);
  if (q->D == 128) {
    bwd_prep_kernel<128><<<n_q, 128, 0, cs>>>(p);
  } else {
    bwd_prep_kernel<64><<<n_q, 128, 0, cs>>>(p);
  }
  if ((s = launched()) != LCSA_OK) return s;
  bwd_lists_kernel<<<static_cast<unsigned>((static_cast<int64_t>(n_k) * 32 + 255) / 256), 256, 0, cs>>>(p);
  if ((s = launched()) != LCSA_OK) return s;
  if (q->D == 128) {
    bwd_dq_kernel<128><<<n_q, BWD_THREADS, BwdLayout<128>::SMEM_DQ, cs>>>(tq, tdo, tk, tv, p);
    if ((s = launched()) != LCSA_OK) return s;
    bwd_dkdv_kernel<128><<<n_k, BWD_THREADS, BwdLayout<128>::SMEM_KV, cs>>>(tq, tdo, tk, tv, p);
  } else {
    bwd_dq_kernel<64><<<n_q, BWD_THREADS, BwdLayout<64>::SMEM_DQ, cs>>>(tq, tdo, tk, tv, p);
    if ((s = launched()) != LCSA_OK) return s;
    bwd_dkdv_kernel<64><<<n_k, BWD_THREADS, BwdLayout<64>::SMEM_KV, cs>>>(tq, tdo, tk, tv, p);
  }
  return launched();
}

// Device addresses of lcsa_select_scratch, looked up once per device.
static std::mutex g_scratch_mu;
static void* g_scratch_ptr[64] = {};

lcsa_status lcsa_select_blocks_noalloc(const double* q_pool, int32_t q_frames, const lcsa_kv_cache* kv,
                                       const lcsa_select_params* sp, int32_t* blk_idx, int32_t* blk_cnt,
                                       lcsa_stream_t stream) {
  if (q_pool == nullptr || kv == nullptr || sp == nullptr || blk_idx == nullptr || blk_cnt == nullptr)
    return LCSA_ERR_INVALID_ARG;
  if (lcsa_select_workspace_bytes(kv, q_frames) > LCSA_SELECT_STATIC_SCRATCH_BYTES)
    return LCSA_ERR_SCRATCH_LIMIT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LCSA_ERR_CUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* ptr = nullptr;  // this device is current: the address is its copy's
      if (cudaGetSymbolAddress(&ptr, lcsa_select_scratch) != cudaSuccess || ptr == nullptr)
        return LCSA_ERR_CUDA;
      g_scratch_ptr[dev] = ptr;
    }
    scratch = g_scratch_ptr[dev];
  }
  // the same validation, kernels and results as the workspace entry point
  return lcsa_select_blocks(q_pool, q_frames, kv, sp, blk_idx, blk_cnt, scratch,
                            LCSA_SELECT_STATIC_SCRATCH_BYTES, stream);
}

static lcsa_status attn_fwd_impl(const lcsa_tensor* q, const lcsa_kv_cache* kv, const int32_t* blk_idx,
                                 const int32_t* blk_cnt, int32_t kmax, int32_t window, int32_t window_mode,
                                 lcsa_tensor* o, float* lse, void* workspace, size_t workspace_bytes,
                                 lcsa_stream_t stream) {
  lcsa_status s = check_tensor(q);
  if (s != LCSA_OK) return s;
  if ((s = check_cache(kv)) != LCSA_OK) return s;
  if (o == nullptr) return LCSA_ERR_INVALID_ARG;
  if ((s = check_tensor(o)) != LCSA_OK) return s;
  if (blk_idx == nullptr || blk_cnt == nullptr || kmax < 1) return LCSA_ERR_INVALID_ARG;
  if (q->B != kv->B || q->H != kv->H || q->Y != kv->Y || q->X != kv->X || q->D != kv->D)
    return LCSA_ERR_SHAPE;
  if (o->B != q->B || o->H != q->H || o->T != q->T || o->Y != q->Y || o->X != q->X || o->D != q->D)
    return LCSA_ERR_SHAPE;
  for (int b = 0; b < kv->B; ++b)
    if (kv->end[b] - kv->begin[b] < 1) return LCSA_ERR_SHAPE;
  // key block ids lie below (cap / 2) * Hb * Wb; the kernel splits them with a
  // float reciprocal (SmallDiv) that is exact below 2^22
  if (static_cast<int64_t>(kv->cap_frames / 2) * (kv->Y / 8) * (kv->X / 8) >= (int64_t{1} << 22))
    return LCSA_ERR_SHAPE;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LCSA_ERR_ALIGN;
  int dev;
  unsigned int* err;
  if ((s = device_setup(&dev, &err)) != LCSA_OK) return s;
  CUtensorMap tq, tk, tv;
  const int64_t cs_x = kv->D, cs_y = static_cast<int64_t>(kv->X) * kv->D;
  const int64_t cs_t = cs_y * kv->Y, cs_h = cs_t * kv->cap_frames;
  if ((s = encode_map(&tq, q->data, q->B, q->H, q->T, q->Y, q->X, q->D, q->stride_h, q->stride_t,
                      q->stride_y, q->stride_x)) != LCSA_OK ||
      (s = encode_map(&tk, kv->k, kv->B, kv->H, kv->cap_frames, kv->Y, kv->X, kv->D, cs_h, cs_t, cs_y,
                      cs_x)) != LCSA_OK ||
      (s = encode_map(&tv, kv->v, kv->B, kv->H, kv->cap_frames, kv->Y, kv->X, kv->D, cs_h, cs_t, cs_y,
                      cs_x)) != LCSA_OK)
    return s;
  AttnParams p{};
  p.blk_idx = blk_idx;
  p.blk_cnt = blk_cnt;
  p.o = static_cast<__nv_bfloat16*>(o->data);
  p.lse = lse;
  p.osh = o->stride_h; p.ost = o->stride_t; p.osy = o->stride_y; p.osx = o->stride_x;
  p.H = q->H; p.Tq = q->T; p.Y = q->Y; p.X = q->X; p.Hb = q->Y / 8; p.Wb = q->X / 8;
  p.nQT = temporal_blocks(q->T);
  p.nQB = p.nQT * p.Hb * p.Wb;
  p.kmax = kmax;
  p.cap = kv->cap_frames;
  p.win = window;
  p.win_mode = window_mode;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(q->D)));
  p.wait_limit_ns = g_wait_limit_ns;
  p.err = err;
  for (int b = 0; b < kv->B; ++b) {
    const int64_t base = ring_base(kv->begin[b], kv->cap_frames);
    p.kv_begin[b] = kv->begin[b] - base;
    p.kv_end[b] = kv->end[b] - base;
  }
  const int64_t units = static_cast<int64_t>(q->B) * q->H * p.nQB;  // one CTA per query block
  if (units > 0x7fffffff / 2) return LCSA_ERR_SHAPE;
  if (units == 0) return LCSA_OK;
  // With a workspace, a last wave that would leave most SMs idle is evened
  // out: its r units run as 2r half-units (the kept blocks split in two) and a
  // merge kernel combines each pair.
  const int64_t sms = g_sm_count[dev];
  const int64_t r = units % sms;
  int64_t grid = units;
  p.split_from = 0x7fffffff;
  if (workspace != nullptr && units > sms && r > 0 && 2 * r <= sms && r <= LCSA_ATTN_SPLIT_MAX &&
      workspace_bytes >= static_cast<size_t>(2 * r * 128 * (q->D + 1) * 4) && aligned16(workspace)) {
    p.split_from = static_cast<int32_t>(units - r);
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = p.part_o + 2 * r * 128 * q->D;
    grid = units + r;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (q->D == 128)
    attn_fwd_kernel<128><<<static_cast<unsigned>(grid), ATTN_THREADS, AttnLayout<128>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
  else
    attn_fwd_kernel<64><<<static_cast<unsigned>(grid), ATTN_THREADS, AttnLayout<64>::SMEM_BYTES, cs>>>(tq, tk, tv, p);
  if ((s = launched()) != LCSA_OK || grid == units) return s;
  const unsigned mgrid = static_cast<unsigned>((r * 128 * 32 + 255) / 256);
  if (q->D == 128) attn_merge_kernel<128><<<mgrid, 256, 0, cs>>>(p, static_cast<int32_t>(r));
  else attn_merge_kernel<64><<<mgrid, 256, 0, cs>>>(p, static_cast<int32_t>(r));
  return launched();
}

lcsa_status lcsa_sparse_attn_fwd(const lcsa_tensor* q, const lcsa_kv_cache* kv, const int32_t* blk_idx,
                                 const int32_t* blk_cnt, int32_t kmax, lcsa_tensor* o, float* lse,
                                 lcsa_stream_t stream) {
  return attn_fwd_impl(q, kv, blk_idx, blk_cnt, kmax, 0, LCSA_WINDOW_TRUNCATE_TOKENS, o, lse, nullptr, 0, stream);
}

lcsa_status lcsa_sparse_attn_fwd_window(const lcsa_tensor* q, const lcsa_kv_cache* kv, const int32_t* blk_idx,
                                        const int32_t* blk_cnt, int32_t kmax, int32_t window, int32_t window_mode,
                                        lcsa_tensor* o, float* lse, lcsa_stream_t stream) {
  if (window < 0 || (window > 0 && window_mode != LCSA_WINDOW_TRUNCATE_TOKENS &&
                     window_mode != LCSA_WINDOW_PRESERVE_TOKENS))
    return LCSA_ERR_INVALID_ARG;
  return attn_fwd_impl(q, kv, blk_idx, blk_cnt, kmax, window, window_mode, o, lse, nullptr, 0, stream);
}

size_t lcsa_sparse_attn_fwd_workspace_bytes(int32_t head_dim) {
  if (head_dim != 64 && head_dim != 128) return 0;
  return static_cast<size_t>(2) * LCSA_ATTN_SPLIT_MAX * 128 * (head_dim + 1) * 4;
}

lcsa_status lcsa_sparse_attn_fwd_ex(const lcsa_tensor* q, const lcsa_kv_cache* kv, const int32_t* blk_idx,
                                    const int32_t* blk_cnt, int32_t kmax, int32_t window, int32_t window_mode,
                                    lcsa_tensor* o, float* lse, void* workspace, size_t workspace_bytes,
                                    lcsa_stream_t stream) {
  if (window < 0 || (window > 0 && window_mode != LCSA_WINDOW_TRUNCATE_TOKENS &&
                     window_mode != LCSA_WINDOW_PRESERVE_TOKENS))
    return LCSA_ERR_INVALID_ARG;
  return attn_fwd_impl(q, kv, blk_idx, blk_cnt, kmax, window, window > 0 ? window_mode : LCSA_WINDOW_TRUNCATE_TOKENS,
                       o, lse, workspace, workspace_bytes, stream);
}

lcsa_status lcsa_last_device_error(lcsa_stream_t stream) {
  int dev;
  unsigned int* err;
  lcsa_status s = device_setup(&dev, &err);
  if (s != LCSA_OK) return s;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return LCSA_ERR_CUDA;
  if (cudaMemcpyAsync(&word, err, sizeof(word), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaMemsetAsync(err, 0, sizeof(word), cs) != cudaSuccess || cudaStreamSynchronize(cs) != cudaSuccess)
    return LCSA_ERR_CUDA;
  if (word & DEVERR_TIMEOUT) return LCSA_ERR_TIMEOUT;
  if (word & DEVERR_BOUNDS) return LCSA_ERR_DEVICE_BOUNDS;
  return LCSA_OK;
}

lcsa_status lcsa_debug_stalled_wait(uint64_t limit_ns, lcsa_stream_t stream) {
  int dev;
  unsigned int* err;
  lcsa_status s = device_setup(&dev, &err);
  if (s != LCSA_OK) return s;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return LCSA_ERR_INVALID_ARG;
  stalled_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, err);
  return launched();
}

lcsa_status lcsa_debug_exp2_poly(const float* x, float* y, int64_t n, lcsa_stream_t stream) {
  if (x == nullptr || y == nullptr || n < 1) return LCSA_ERR_INVALID_ARG;
  int dev;
  unsigned int* err;
  lcsa_status s = device_setup(&dev, &err);
  if (s != LCSA_OK) return s;
  const int64_t threads = (n + 1) / 2;
  const int64_t grid = (threads + 255) / 256;
  if (grid > 0x7fffffff) return LCSA_ERR_SHAPE;
  exp2_poly_kernel<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launched();
}

lcsa_status lcsa_debug_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns == 0 ? kDefaultWaitNs : ns;
  return LCSA_OK;
}

}  // extern "C"

#include "pipeline.cuh"
