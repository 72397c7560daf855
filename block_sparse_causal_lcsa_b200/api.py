"""PyTorch-facing binding of liblcsa.so.

Each function takes torch CUDA tensors, marshals their pointers, extents and
strides into the C structs of include/lcsa.h and calls the entry point of the
same name on the current torch stream. Output buffers are allocated with torch
when the caller does not pass them (the library itself allocates nothing,
except the buffers a NativePipeline owns).
No step of the attention path runs here: there is no CPU fallback, and a
missing or incomplete liblcsa.so raises ImportError at import.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _abi

_lib = _abi.load()

OK = _abi.OK
WINDOW_TRUNCATE = _abi.WINDOW_TRUNCATE
WINDOW_PRESERVE = _abi.WINDOW_PRESERVE
WINDOW_TRUNCATE_TOKENS = _abi.WINDOW_TRUNCATE_TOKENS
WINDOW_PRESERVE_TOKENS = _abi.WINDOW_PRESERVE_TOKENS
TIE_EPS = 1e-5


class LcsaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = _lib.lcsa_status_string(status).decode()
        super().__init__("%s: %s (status %d)" % (what, msg, status) if what else msg)


def _check(status: int, what: str) -> None:
    if status != OK:
        raise LcsaError(status, what)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def tensor_desc(x: torch.Tensor) -> _abi.Tensor:
    """lcsa_tensor for a bf16 tensor of shape [B][H][T][Y][X][D] (D unit stride)."""
    if x.dim() != 6 or x.dtype != torch.bfloat16 or not x.is_cuda:
        raise ValueError("expected a CUDA bf16 tensor [B][H][T][Y][X][D]")
    if x.stride(5) != 1:
        raise ValueError("the channel dimension must have unit stride")
    B, H, T, Y, X, D = x.shape
    sb, sh, st, sy, sx, _ = x.stride()
    return _abi.Tensor(x.data_ptr(), B, H, T, Y, X, D, sb, sh, st, sy, sx)


def pooled_shape(x: torch.Tensor) -> Tuple[int, ...]:
    B, H, T, Y, X, D = x.shape
    return (B, H, (T + 1) // 2, Y // 8, X // 8, D)


def _check_tokens(name: str, t) -> None:
    """A token tensor [B][H][T][Y][X][D] in bf16 (its device is checked with
    the call's other tensors)."""
    if not isinstance(t, torch.Tensor) or t.dim() != 6 or t.dtype != torch.bfloat16:
        raise ValueError("%s must be a bf16 tensor [B][H][T][Y][X][D]" % name)


def _check_buffer(name: str, t, dtype: torch.dtype, shape) -> None:
    """A buffer the library takes as a bare pointer and sizes from its other
    arguments: any other dtype, shape or layout would let a kernel read or
    write past it (ValueError, nothing launched)."""
    if not isinstance(t, torch.Tensor):
        raise ValueError("%s must be a tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _check_workspace(t) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor")


def _check_device(dev: torch.device, **tensors) -> None:
    """All tensors of a call in the memory of the one GPU it runs on (the
    kernels dereference their pointers there). None entries are skipped."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor, got %s" % (name, t.device))
        if t.device != dev:
            raise ValueError("%s must be on %s with the call's other tensors, got %s" % (name, dev, t.device))


def _query_blocks(q: torch.Tensor) -> int:
    _, _, T, Y, X, _ = q.shape
    return ((T + 1) // 2) * (Y // 8) * (X // 8)


def _check_block_lists(q: torch.Tensor, blk_idx, blk_cnt) -> None:
    """blk_idx int32 [B,H,nQB,kmax] and blk_cnt int32 [B,H,nQB] for the query
    chunk q (nQB = ceil(T/2) * Y/8 * X/8); kmax is blk_idx's last extent."""
    if not isinstance(blk_idx, torch.Tensor) or blk_idx.dim() != 4:
        raise ValueError("blk_idx must be an int32 tensor [B,H,nQB,kmax]")
    B, H = q.shape[0], q.shape[1]
    nQB = _query_blocks(q)
    _check_buffer("blk_idx", blk_idx, torch.int32, (B, H, nQB, blk_idx.shape[-1]))
    _check_buffer("blk_cnt", blk_cnt, torch.int32, (B, H, nQB))


def pool_qk(q: torch.Tensor, k: Optional[torch.Tensor] = None,
            q_pool: Optional[torch.Tensor] = None, k_pool: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None):
    """Mean-pool Q (and K) over 2x8x8 token blocks into float64 features."""
    _check_tokens("q", q)
    if k is not None:
        _check_tokens("k", k)
    if q_pool is None:
        q_pool = torch.empty(pooled_shape(q), dtype=torch.float64, device=q.device)
    else:
        _check_buffer("q_pool", q_pool, torch.float64, pooled_shape(q))
    if k is not None and k_pool is None:
        k_pool = torch.empty(pooled_shape(k), dtype=torch.float64, device=k.device)
    elif k is not None:
        _check_buffer("k_pool", k_pool, torch.float64, pooled_shape(k))
    _check_device(q.device, q=q, k=k, q_pool=q_pool, k_pool=k_pool if k is not None else None)
    qd = tensor_desc(q)
    kd = tensor_desc(k) if k is not None else None
    _check(_lib.lcsa_pool_qk(C.byref(qd), C.byref(kd) if kd is not None else None,
                             q_pool.data_ptr(), k_pool.data_ptr() if k is not None else None,
                             _stream(stream)), "lcsa_pool_qk")
    return q_pool, k_pool


class KVCache:
    """Streaming ring cache of K, V and pooled K for B streams (device buffers
    owned by this object, begin/end state kept host-side in the C struct)."""

    def __init__(self, B: int, H: int, cap_frames: int, Y: int, X: int, D: int,
                 device="cuda", k: torch.Tensor = None, v: torch.Tensor = None,
                 k_pool: torch.Tensor = None):
        shape = (B, H, cap_frames, Y, X, D)
        self.k = k if k is not None else torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.v = v if v is not None else torch.empty(shape, dtype=torch.bfloat16, device=device)
        self.k_pool = (k_pool if k_pool is not None else
                       torch.empty((B, H, cap_frames // 2, Y // 8, X // 8, D), dtype=torch.float64,
                                   device=device))
        pool_shape = (B, H, cap_frames // 2, Y // 8, X // 8, D)
        for name, t, dtype, shp in (("k", self.k, torch.bfloat16, shape), ("v", self.v, torch.bfloat16, shape),
                                    ("k_pool", self.k_pool, torch.float64, pool_shape)):
            _check_buffer(name, t, dtype, shp)
            if t.device != self.k.device:
                raise ValueError("k, v and k_pool must be on one device")
        self.struct = _abi.KVCacheStruct()
        self.struct.k = self.k.data_ptr()
        self.struct.v = self.v.data_ptr()
        self.struct.k_pool = self.k_pool.data_ptr()
        self.struct.B, self.struct.H, self.struct.cap_frames = B, H, cap_frames
        self.struct.Y, self.struct.X, self.struct.D = Y, X, D
        self.B, self.H, self.cap_frames, self.Y, self.X, self.D = B, H, cap_frames, Y, X, D

    @classmethod
    def wrap(cls, k: torch.Tensor, v: torch.Tensor, k_pool: torch.Tensor) -> "KVCache":
        """View whole K/V sequences [B][H][F][Y][X][D] (F even) as a full cache."""
        B, H, F, Y, X, D = k.shape
        c = cls(B, H, F, Y, X, D, k=k.contiguous(), v=v.contiguous(), k_pool=k_pool.contiguous())
        for b in range(B):
            c.struct.begin[b] = 0
            c.struct.end[b] = F
        return c

    def begin(self, b: int) -> int:
        return int(self.struct.begin[b])

    def end(self, b: int) -> int:
        return int(self.struct.end[b])

    def frames(self, b: int) -> int:
        return self.end(b) - self.begin(b)

    def reset(self) -> None:
        for b in range(self.B):
            self.struct.begin[b] = 0
            self.struct.end[b] = 0

    def state(self):
        return [(self.begin(b), self.end(b)) for b in range(self.B)]

    def set_state(self, state) -> None:
        for b, (lo, hi) in enumerate(state):
            self.struct.begin[b] = lo
            self.struct.end[b] = hi


def kv_append(cache: KVCache, k_new: torch.Tensor, v_new: torch.Tensor,
              k_pool_new: Optional[torch.Tensor] = None, stream_offset: int = 0,
              stream: Optional[torch.cuda.Stream] = None) -> None:
    """Append a chunk to streams [offset, offset+B) of the cache. Without
    k_pool_new the call pools K itself while copying it (one read of K)."""
    _check_tokens("k_new", k_new)
    _check_tokens("v_new", v_new)
    if k_pool_new is not None:
        _check_buffer("k_pool_new", k_pool_new, torch.float64, pooled_shape(k_new))
    _check_device(cache.k.device, cache=cache.k, k_new=k_new, v_new=v_new, k_pool_new=k_pool_new)
    kd, vd = tensor_desc(k_new), tensor_desc(v_new)
    _check(_lib.lcsa_kv_append(C.byref(cache.struct), C.byref(kd), C.byref(vd),
                               k_pool_new.data_ptr() if k_pool_new is not None else None,
                               stream_offset, _stream(stream)),
           "lcsa_kv_append")


def ingest_chunk(q: torch.Tensor, cache: KVCache, k_new: torch.Tensor, v_new: torch.Tensor,
                 q_pool: Optional[torch.Tensor] = None, stream_offset: int = 0,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """pool_qk(q) and kv_append(cache, k_new, v_new) (K pooled on the way) in
    one launch; returns q_pool."""
    _check_tokens("q", q)
    if q_pool is None:
        q_pool = torch.empty(pooled_shape(q), dtype=torch.float64, device=q.device)
    else:
        _check_buffer("q_pool", q_pool, torch.float64, pooled_shape(q))
    _check_tokens("k_new", k_new)
    _check_tokens("v_new", v_new)
    _check_device(cache.k.device, cache=cache.k, q=q, k_new=k_new, v_new=v_new, q_pool=q_pool)
    qd, kd, vd = tensor_desc(q), tensor_desc(k_new), tensor_desc(v_new)
    _check(_lib.lcsa_ingest_chunk(C.byref(qd), q_pool.data_ptr(), C.byref(cache.struct), C.byref(kd), C.byref(vd),
                                  stream_offset, _stream(stream)), "lcsa_ingest_chunk")
    return q_pool


@dataclass
class SelectParams:
    top_k: int = 0
    density: float = 0.0
    window: int = 0
    window_mode: int = WINDOW_TRUNCATE
    tie_eps: float = TIE_EPS

    def struct(self, kmax: int = 0) -> _abi.SelectParamsStruct:
        return _abi.SelectParamsStruct(self.top_k, self.window, self.window_mode, kmax,
                                       float(self.density), float(self.tie_eps))


def select_kmax(cache: KVCache, q_frames: int, params: SelectParams) -> int:
    sp = params.struct()
    return int(_lib.lcsa_select_kmax(C.byref(cache.struct), q_frames, C.byref(sp)))


def select_workspace_bytes(cache: KVCache, q_frames: int) -> int:
    return int(_lib.lcsa_select_workspace_bytes(C.byref(cache.struct), q_frames))


def _check_select_io(q_pool: torch.Tensor, q_frames: int, cache: KVCache, kmax: int,
                     blk_idx: torch.Tensor, blk_cnt: torch.Tensor) -> None:
    """The C call writes blk_idx / blk_cnt and reads q_pool by the cache's
    extents: reject anything whose dtype, shape, layout or device would let
    the kernels read or write past a tensor (ValueError, nothing launched)."""
    nQT = (q_frames + 1) // 2
    Hb, Wb = cache.Y // 8, cache.X // 8
    nQB = nQT * Hb * Wb
    want = {"q_pool": (q_pool, torch.float64, (cache.B, cache.H, nQT, Hb, Wb, cache.D)),
            "blk_idx": (blk_idx, torch.int32, (cache.B, cache.H, nQB, kmax)),
            "blk_cnt": (blk_cnt, torch.int32, (cache.B, cache.H, nQB))}
    for name, (t, dtype, shape) in want.items():
        _check_buffer(name, t, dtype, shape)
    _check_device(cache.k.device, cache=cache.k, q_pool=q_pool, blk_idx=blk_idx, blk_cnt=blk_cnt)


def select_blocks(q_pool: torch.Tensor, q_frames: int, cache: KVCache, params: SelectParams,
                  kmax: Optional[int] = None, blk_idx: Optional[torch.Tensor] = None,
                  blk_cnt: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None):
    """Top-K key blocks of every query block: (blk_idx [B,H,nQB,kmax], blk_cnt [B,H,nQB])."""
    if kmax is None:
        kmax = blk_idx.shape[-1] if blk_idx is not None else select_kmax(cache, q_frames, params)
    nQB = ((q_frames + 1) // 2) * (cache.Y // 8) * (cache.X // 8)
    dev = q_pool.device
    if blk_idx is None:
        blk_idx = torch.empty((cache.B, cache.H, nQB, kmax), dtype=torch.int32, device=dev)
    if blk_cnt is None:
        blk_cnt = torch.empty((cache.B, cache.H, nQB), dtype=torch.int32, device=dev)
    _check_select_io(q_pool, q_frames, cache, kmax, blk_idx, blk_cnt)
    need = select_workspace_bytes(cache, q_frames)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    else:
        _check_workspace(workspace)
        _check_device(cache.k.device, workspace=workspace)
    sp = params.struct(kmax)
    _check(_lib.lcsa_select_blocks(q_pool.data_ptr(), q_frames, C.byref(cache.struct), C.byref(sp),
                                   blk_idx.data_ptr(), blk_cnt.data_ptr(), workspace.data_ptr(),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "lcsa_select_blocks")
    return blk_idx, blk_cnt


def select_blocks_noalloc(q_pool: torch.Tensor, q_frames: int, cache: KVCache, params: SelectParams,
                          blk_idx: torch.Tensor, blk_cnt: torch.Tensor,
                          stream: Optional[torch.cuda.Stream] = None):
    """select_blocks into caller-given outputs, with the library's fixed
    scratch array in place of a workspace: nothing is allocated, so it suits
    callers that may not allocate device memory while they run. kmax is
    blk_idx.shape[-1]; q_pool must be float64 [B,H,nQT,Y/8,X/8,D] and the
    outputs int32 [B,H,nQB,kmax] / [B,H,nQB] on the cache's device (else
    ValueError). Raises LcsaError(ERR_SCRATCH_LIMIT) when the selection needs
    more than SELECT_STATIC_SCRATCH_BYTES of scratch; calls that overlap on
    the GPU share that scratch and must be serialised."""
    if not isinstance(blk_idx, torch.Tensor) or blk_idx.dim() != 4:
        raise ValueError("blk_idx must be an int32 tensor [B,H,nQB,kmax]")
    _check_select_io(q_pool, q_frames, cache, blk_idx.shape[-1], blk_idx, blk_cnt)
    sp = params.struct(blk_idx.shape[-1])
    _check(_lib.lcsa_select_blocks_noalloc(q_pool.data_ptr(), q_frames, C.byref(cache.struct),
                                           C.byref(sp), blk_idx.data_ptr(), blk_cnt.data_ptr(),
                                           _stream(stream)),
           "lcsa_select_blocks_noalloc")
    return blk_idx, blk_cnt


def sparse_attn_fwd(q: torch.Tensor, cache: KVCache, blk_idx: torch.Tensor, blk_cnt: torch.Tensor,
                    o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                    with_lse: bool = True, stream: Optional[torch.cuda.Stream] = None,
                    window: int = 0, window_mode: int = WINDOW_TRUNCATE_TOKENS,
                    workspace: Optional[torch.Tensor] = None):
    """Attention of the query chunk over its kept key blocks: (O bf16 like q, LSE fp32).
    With ``window`` > 0 (a token-level window mode), each query token only sees
    the key tokens inside its window. With a ``workspace`` (see
    attn_workspace), a partly empty last wave of CTAs is evened out by splitting
    its query blocks in two (lcsa_sparse_attn_fwd_ex)."""
    _check_tokens("q", q)
    if o is None:
        o = torch.empty_like(q)
    _check_tokens("o", o)
    if lse is None and with_lse:
        lse = torch.empty(q.shape[:5], dtype=torch.float32, device=q.device)
    _check_block_lists(q, blk_idx, blk_cnt)
    if lse is not None:
        _check_buffer("lse", lse, torch.float32, q.shape[:5])
    if workspace is not None:
        _check_workspace(workspace)
    _check_device(q.device, q=q, cache=cache.k, o=o, lse=lse, blk_idx=blk_idx, blk_cnt=blk_cnt, workspace=workspace)
    qd, od = tensor_desc(q), tensor_desc(o)
    lse_ptr = lse.data_ptr() if lse is not None else None
    if workspace is not None:
        _check(_lib.lcsa_sparse_attn_fwd_ex(C.byref(qd), C.byref(cache.struct), blk_idx.data_ptr(),
                                            blk_cnt.data_ptr(), blk_idx.shape[-1], window, window_mode,
                                            C.byref(od), lse_ptr, workspace.data_ptr(),
                                            workspace.numel() * workspace.element_size(), _stream(stream)),
               "lcsa_sparse_attn_fwd_ex")
    elif window > 0:
        _check(_lib.lcsa_sparse_attn_fwd_window(C.byref(qd), C.byref(cache.struct), blk_idx.data_ptr(),
                                                blk_cnt.data_ptr(), blk_idx.shape[-1], window, window_mode,
                                                C.byref(od), lse_ptr, _stream(stream)),
               "lcsa_sparse_attn_fwd_window")
    else:
        _check(_lib.lcsa_sparse_attn_fwd(C.byref(qd), C.byref(cache.struct), blk_idx.data_ptr(),
                                         blk_cnt.data_ptr(), blk_idx.shape[-1], C.byref(od), lse_ptr,
                                         _stream(stream)),
               "lcsa_sparse_attn_fwd")
    return o, lse


def attn_workspace(head_dim: int, device="cuda") -> torch.Tensor:
    """Workspace for sparse_attn_fwd's tail split (lcsa_sparse_attn_fwd_workspace_bytes)."""
    n = int(_lib.lcsa_sparse_attn_fwd_workspace_bytes(head_dim))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def segment_blocks(q_frames: int, cache: KVCache, kmax: Optional[int] = None,
                   blk_idx: Optional[torch.Tensor] = None, blk_cnt: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None):
    """Block lists for dense attention inside each stream (segment) of the cache:
    (blk_idx [B,H,nQB,kmax], blk_cnt [B,H,nQB]) for sparse_attn_fwd / _bwd."""
    if blk_idx is not None:
        if not isinstance(blk_idx, torch.Tensor) or blk_idx.dim() != 4:
            raise ValueError("blk_idx must be an int32 tensor [B,H,nQB,kmax]")
        if kmax is not None and kmax != blk_idx.shape[-1]:
            raise ValueError("kmax %d differs from blk_idx's last extent %d" % (kmax, blk_idx.shape[-1]))
        kmax = blk_idx.shape[-1]
    if kmax is None:
        kmax = int(_lib.lcsa_segment_kmax(C.byref(cache.struct)))
    nQB = ((q_frames + 1) // 2) * (cache.Y // 8) * (cache.X // 8)
    dev = cache.k.device
    if blk_idx is None:
        blk_idx = torch.empty((cache.B, cache.H, nQB, kmax), dtype=torch.int32, device=dev)
    if blk_cnt is None:
        blk_cnt = torch.empty((cache.B, cache.H, nQB), dtype=torch.int32, device=dev)
    _check_buffer("blk_idx", blk_idx, torch.int32, (cache.B, cache.H, nQB, kmax))
    _check_buffer("blk_cnt", blk_cnt, torch.int32, (cache.B, cache.H, nQB))
    _check_device(dev, cache=cache.k, blk_idx=blk_idx, blk_cnt=blk_cnt)
    _check(_lib.lcsa_segment_blocks(q_frames, C.byref(cache.struct), blk_idx.shape[-1], blk_idx.data_ptr(),
                                    blk_cnt.data_ptr(), _stream(stream)), "lcsa_segment_blocks")
    return blk_idx, blk_cnt


def sparse_attn_bwd_workspace_bytes(cache: KVCache, q_frames: int) -> int:
    return int(_lib.lcsa_sparse_attn_bwd_workspace_bytes(C.byref(cache.struct), q_frames))


def sparse_attn_bwd(q: torch.Tensor, cache: KVCache, blk_idx: torch.Tensor, blk_cnt: torch.Tensor,
                    o: torch.Tensor, lse: torch.Tensor, d_o: torch.Tensor,
                    dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                    dv: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None):
    """Gradients of sparse_attn_fwd for the same selection: (dq like q, dk and
    dv in the cache layout [B][H][cap][Y][X][D]). dk / dv default to zeros, so
    ring slots outside the cached frames read as zero."""
    for name, t in (("q", q), ("o", o), ("d_o", d_o)):
        _check_tokens(name, t)
    if dq is None:
        dq = torch.empty_like(q)
    _check_tokens("dq", dq)
    if dk is None:
        dk = torch.zeros_like(cache.k)
    if dv is None:
        dv = torch.zeros_like(cache.v)
    _check_block_lists(q, blk_idx, blk_cnt)
    _check_buffer("lse", lse, torch.float32, q.shape[:5])
    _check_buffer("dk", dk, torch.bfloat16, cache.k.shape)
    _check_buffer("dv", dv, torch.bfloat16, cache.v.shape)
    if workspace is None:
        need = sparse_attn_bwd_workspace_bytes(cache, q.shape[2])
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check_workspace(workspace)
    _check_device(q.device, q=q, cache=cache.k, o=o, d_o=d_o, dq=dq, lse=lse, dk=dk, dv=dv, blk_idx=blk_idx,
                  blk_cnt=blk_cnt, workspace=workspace)
    qd, od, gd, dqd = tensor_desc(q), tensor_desc(o), tensor_desc(d_o), tensor_desc(dq)
    _check(_lib.lcsa_sparse_attn_bwd(C.byref(qd), C.byref(cache.struct), blk_idx.data_ptr(), blk_cnt.data_ptr(),
                                     blk_idx.shape[-1], C.byref(od), lse.data_ptr(), C.byref(gd), C.byref(dqd),
                                     dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "lcsa_sparse_attn_bwd")
    return dq, dk, dv


def last_device_error(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronise the stream, read and clear the device error word (status code)."""
    return int(_lib.lcsa_last_device_error(_stream(stream)))


def debug_stalled_wait(limit_ns: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    _check(_lib.lcsa_debug_stalled_wait(limit_ns, _stream(stream)), "lcsa_debug_stalled_wait")


def debug_exp2_poly(x: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """2^x through the attention kernel's FMA-pipe polynomial (test hook)."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous CUDA float32 tensor")
    y = torch.empty_like(x)
    _check(_lib.lcsa_debug_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(), _stream(stream)),
           "lcsa_debug_exp2_poly")
    return y


def debug_set_wait_limit_ns(ns: int) -> None:
    _check(_lib.lcsa_debug_set_wait_limit_ns(ns), "lcsa_debug_set_wait_limit_ns")


class StreamingStep:
    """One streaming LCSA step over preallocated buffers: pool Q, append K/V to
    the cache (pooling K on the way), select the top-K blocks, attend.

    The four library calls are the whole step; buffers are allocated once here
    so that repeated steps launch kernels only.
    """

    def __init__(self, cache: KVCache, q_frames: int, params: SelectParams):
        self.cache = cache
        self.q_frames = q_frames
        self.params = params
        dev = cache.k.device
        B, H, Y, X, D = cache.B, cache.H, cache.Y, cache.X, cache.D
        nQT = (q_frames + 1) // 2
        self.q_pool = torch.empty((B, H, nQT, Y // 8, X // 8, D), dtype=torch.float64, device=dev)
        # capacity for the fullest cache state this step can see
        full = _abi.KVCacheStruct.from_buffer_copy(cache.struct)
        for b in range(B):
            full.begin[b], full.end[b] = 0, cache.cap_frames
        sp = params.struct()
        self.kmax = int(_lib.lcsa_select_kmax(C.byref(full), q_frames, C.byref(sp)))
        ws = int(_lib.lcsa_select_workspace_bytes(C.byref(full), q_frames))
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        nQB = nQT * (Y // 8) * (X // 8)
        self.blk_idx = torch.empty((B, H, nQB, self.kmax), dtype=torch.int32, device=dev)
        self.blk_cnt = torch.empty((B, H, nQB), dtype=torch.int32, device=dev)
        self.o = torch.empty((B, H, q_frames, Y, X, D), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((B, H, q_frames, Y, X), dtype=torch.float32, device=dev)
        self.attn_ws = attn_workspace(D, dev)
        self._static = None
        self._graphs = {}

    def graph_step(self, q: Optional[torch.Tensor] = None, k_new: Optional[torch.Tensor] = None,
                   v_new: Optional[torch.Tensor] = None):
        """The same step replayed from a CUDA graph: the inputs are copied into
        static buffers (without inputs, the buffers are used as they are: the
        caller may have written the chunk there), then one graph launch runs
        pool, append, select and attention. The library passes frame numbers to its kernels modulo the
        ring capacity, so a stream in steady state needs one graph per ring
        phase; each is captured the first time its phase comes up (make that
        first step an ordinary one outside any timing). Returns (o, lse), the
        step's static output buffers."""
        if self._static is None:
            if q is None:
                raise ValueError("the first graph_step needs the chunk")
            self._static = (torch.empty_like(q), torch.empty_like(k_new), torch.empty_like(v_new))
            self._graphs = {}
        sq, sk, sv = self._static
        if q is not None:
            sq.copy_(q)
            sk.copy_(k_new)
            sv.copy_(v_new)
        cap = self.cache.cap_frames
        key = tuple((b % cap, e - b) for b, e in self.cache.state())
        g = self._graphs.get(key)
        if g is None:
            saved = self.cache.state()
            self(sq, sk, sv)                  # device set-up and a warm run outside the capture
            torch.cuda.synchronize()
            self.cache.set_state(saved)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self(sq, sk, sv)
            self.cache.set_state(saved)       # the capture advanced the host state without running
            self._graphs[key] = g
        g.replay()
        _check(_lib.lcsa_kv_advance(C.byref(self.cache.struct), sk.shape[2], sk.shape[0], 0), "lcsa_kv_advance")
        return self.o, self.lse

    def __call__(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                 stream: Optional[torch.cuda.Stream] = None):
        ingest_chunk(q, self.cache, k_new, v_new, self.q_pool, 0, stream)
        select_blocks(self.q_pool, self.q_frames, self.cache, self.params, self.kmax,
                      self.blk_idx, self.blk_cnt, self.workspace, stream)
        tw = self.params.window if self.params.window_mode >= WINDOW_TRUNCATE_TOKENS else 0
        sparse_attn_fwd(q, self.cache, self.blk_idx, self.blk_cnt, self.o, self.lse, stream=stream,
                        window=tw, window_mode=self.params.window_mode, workspace=self.attn_ws)
        return self.o, self.lse


class NativePipeline:
    """The library's streaming pipeline (lcsa_pipeline_*): chunks of Q, K, V
    from pinned host tensors, the step (ingest, select, attention) and O back
    to a pinned host tensor, with the copies of one chunk overlapping the
    steps of its neighbours, all queued by the C library on its own streams.
    It owns its device buffers and advances `cache` (whose state it shares)
    chunk by chunk. Host tensors must stay untouched until `sync()`."""

    def __init__(self, cache: "KVCache", q_frames: int, params: SelectParams):
        self.cache = cache          # the pipeline holds a pointer to cache.struct
        self.shape = (cache.B, cache.H, q_frames, cache.Y, cache.X, cache.D)
        h = C.c_void_p()
        _check(_lib.lcsa_pipeline_create(C.byref(cache.struct), q_frames, C.byref(params.struct()), C.byref(h)),
               "lcsa_pipeline_create")
        self._h = h

    def submit(self, hq: torch.Tensor, hk: torch.Tensor, hv: torch.Tensor, ho: torch.Tensor) -> None:
        for t in (hq, hk, hv, ho):
            if t.is_cuda or not t.is_pinned() or not t.is_contiguous() or t.dtype != torch.bfloat16:
                raise ValueError("NativePipeline takes contiguous pinned bf16 host tensors")
            if tuple(t.shape) != self.shape:
                raise ValueError("expected host tensors of shape %s" % (self.shape,))
        _check(_lib.lcsa_pipeline_submit(self._h, hq.data_ptr(), hk.data_ptr(), hv.data_ptr(), ho.data_ptr()),
               "lcsa_pipeline_submit")

    def sync(self) -> None:
        _check(_lib.lcsa_pipeline_sync(self._h), "lcsa_pipeline_sync")

    def start_timer(self) -> None:
        _check(_lib.lcsa_pipeline_start_timer(self._h), "lcsa_pipeline_start_timer")

    def elapsed_ms(self) -> float:
        ms = C.c_float()
        _check(_lib.lcsa_pipeline_elapsed_ms(self._h, C.byref(ms)), "lcsa_pipeline_elapsed_ms")
        return float(ms.value)

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.lcsa_pipeline_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()


class HostPipeline:
    """Streams chunks from pinned host memory through a StreamingStep, with the
    copies of one chunk overlapping the compute of its neighbours (a streaming
    video stage receives frames from the host and returns them there).

    Host-to-device copies run on their own stream into two alternating device
    input sets; the step runs on the caller's current stream once its inputs
    have landed; the device-to-host copy of O runs on a third stream. Inputs
    of chunk i+1 therefore cross PCIe while chunk i computes and chunk i-1's
    output travels back. All ordering is by CUDA events; nothing blocks the
    host. `submit` returns the event that completes when O is in `ho`.
    """

    def __init__(self, step: StreamingStep):
        self.step = step
        self.h2d_stream = torch.cuda.Stream(device=step.o.device)
        self.d2h_stream = torch.cuda.Stream(device=step.o.device)
        self._bufs = None
        self._in_ready = [torch.cuda.Event(), torch.cuda.Event()]
        self._in_free = [None, None]
        self._out_free = None
        self._n = 0

    def submit(self, hq: torch.Tensor, hk: torch.Tensor, hv: torch.Tensor,
               ho: torch.Tensor) -> torch.cuda.Event:
        for t in (hq, hk, hv, ho):
            if t.is_cuda or not t.is_pinned():
                raise ValueError("HostPipeline takes pinned host tensors")
        if ho.shape != self.step.o.shape or ho.dtype != self.step.o.dtype:
            raise ValueError("ho must match the step's output %s %s" % (tuple(self.step.o.shape), self.step.o.dtype))
        dev = self.step.o.device
        if self._bufs is None:
            self._bufs = [tuple(torch.empty(t.shape, dtype=t.dtype, device=dev) for t in (hq, hk, hv))
                          for _ in range(2)]
        slot = self._n & 1
        dq, dk, dv = self._bufs[slot]
        if dq.shape != hq.shape or dk.shape != hk.shape or dv.shape != hv.shape:
            raise ValueError("chunk shapes must stay the same across submits")
        # inputs: wait until the step that last read this slot has finished
        if self._in_free[slot] is not None:
            self.h2d_stream.wait_event(self._in_free[slot])
        with torch.cuda.stream(self.h2d_stream):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            self._in_ready[slot].record(self.h2d_stream)
        cur = torch.cuda.current_stream(dev)
        cur.wait_event(self._in_ready[slot])
        # O is overwritten by this step: the previous read-back must be done
        if self._out_free is not None:
            cur.wait_event(self._out_free)
        o, _ = self.step(dq, dk, dv)
        computed = torch.cuda.Event()
        computed.record(cur)
        self._in_free[slot] = computed
        self.d2h_stream.wait_event(computed)
        done = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.d2h_stream):
            ho.copy_(o, non_blocking=True)
            done.record(self.d2h_stream)
        self._out_free = done
        self._n += 1
        return done
