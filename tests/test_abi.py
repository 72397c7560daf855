"""The C-ABI library builds for sm_100a, loads without a GPU and exports every
entry point include/*.h declares; argument errors are returned before any
CUDA call. No compute call is made here."""
import ctypes as C
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    # loaded by path: importing the package would load the (possibly stale) library first
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "lcsa_build", os.path.join(ROOT, "block_sparse_causal_lcsa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def lib():
    _build_module().build()
    from block_sparse_causal_lcsa_b200 import _abi

    return _abi.load()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names |= set(re.findall(r"LCSA_API\s+[\w\s\*]+?\b(lcsa_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    from block_sparse_causal_lcsa_b200 import _abi
    assert names == set(_abi.PROTOTYPES), "ctypes prototypes out of sync with the header"


def test_abi_version_and_status_strings(lib):
    assert lib.lcsa_abi_version() == 1
    assert lib.lcsa_status_string(0) == b"ok"
    assert b"timed out" in lib.lcsa_status_string(-7)


def test_struct_layouts_match_header():
    from block_sparse_causal_lcsa_b200 import _abi
    # offsets computed from include/lcsa.h by hand (LP64)
    assert C.sizeof(_abi.Tensor) == 8 + 6 * 4 + 5 * 8
    assert _abi.Tensor.stride_b.offset == 32
    assert C.sizeof(_abi.KVCacheStruct) == 3 * 8 + 6 * 4 + 2 * 64 * 8
    assert _abi.KVCacheStruct.begin.offset == 48
    assert C.sizeof(_abi.SelectParamsStruct) == 4 * 4 + 2 * 8


def test_argument_errors_before_any_launch(lib):
    from block_sparse_causal_lcsa_b200 import _abi
    # null tensors / pointers are rejected before the device is touched
    assert lib.lcsa_pool_qk(None, None, None, None, None) == _abi.ERR_INVALID_ARG
    t = _abi.Tensor(0x1000, 1, 1, 2, 16, 16, 96, 0, 0, 0, 0, 0)
    assert lib.lcsa_pool_qk(C.byref(t), None, 0x2000, None, None) == _abi.ERR_SHAPE  # D = 96
    t.D = 128
    t.stride_x, t.stride_y, t.stride_t, t.stride_h, t.stride_b = 128, 2048, 32768, 65536, 65536
    t.data = 0x1008
    assert lib.lcsa_pool_qk(C.byref(t), None, 0x2000, None, None) == _abi.ERR_ALIGN
    t.data = 0x1000
    t.stride_b = 3 * 65536  # batch and heads must merge
    assert lib.lcsa_pool_qk(C.byref(t), None, 0x2000, None, None) == _abi.ERR_SHAPE
    kv = _abi.KVCacheStruct()
    assert lib.lcsa_kv_append(C.byref(kv), C.byref(t), C.byref(t), None, 0, None) == _abi.ERR_INVALID_ARG
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 1, 5, 16, 16, 128
    sp = _abi.SelectParamsStruct(2, 0, 0, 2, 0.0, 1e-5)
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 1 << 20, None) == _abi.ERR_SHAPE
    kv.cap_frames = 6
    kv.end[0] = 3  # end must stay even
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 1 << 20, None) == _abi.ERR_INVALID_ARG
    kv.end[0] = 6
    sp.window = 4  # even window
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 1 << 20, None) == _abi.ERR_INVALID_ARG
    sp.window = 0
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 8, None) == _abi.ERR_WORKSPACE
    sp.kmax = 1  # K = 2 does not fit
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 1 << 20, None) == _abi.ERR_CAPACITY
    # more than 2048 causal candidates per query block: 513 temporal blocks x 4
    sp.kmax = 2
    kv.cap_frames, kv.end[0] = 1026, 1026
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, 1 << 40, None) == _abi.ERR_SHAPE


def test_attention_rejects_caches_of_2_22_key_blocks(lib):
    """Key block ids are split in the kernel with a float reciprocal that is
    exact below 2^22: a cache of (cap/2) * Hb * Wb >= 2^22 key blocks is an
    LCSA_ERR_SHAPE before any device work (the pointers here are never used)."""
    from block_sparse_causal_lcsa_b200 import _abi
    t = _abi.Tensor(0x1000, 1, 1, 2, 64, 64, 128, 0, 0, 0, 0, 0)
    t.stride_x, t.stride_y, t.stride_t = 128, 64 * 128, 64 * 64 * 128
    t.stride_h = t.stride_b = 2 * t.stride_t
    kv = _abi.KVCacheStruct()
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.Y, kv.X, kv.D = 1, 1, 64, 64, 128
    kv.cap_frames = 2 * (1 << 16)                    # 2^16 temporal blocks x 64 spatial = 2^22
    kv.begin[0], kv.end[0] = 0, 2
    args = (C.byref(t), C.byref(kv), 0x5000, 0x6000, 1, C.byref(t), None, None)
    assert lib.lcsa_sparse_attn_fwd(*args) == _abi.ERR_SHAPE


def test_pipeline_argument_errors(lib):
    """lcsa_pipeline_* reject bad arguments before any device allocation or
    copy (only invalid requests here: a valid one would allocate)."""
    from block_sparse_causal_lcsa_b200 import _abi
    kv = _abi.KVCacheStruct()
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 1, 6, 16, 16, 128
    sp = _abi.SelectParamsStruct(0, 0, 0, 0, 0.136, 1e-5)
    h = C.c_void_p(0x1)
    assert lib.lcsa_pipeline_create(C.byref(kv), 2, C.byref(sp), None) == _abi.ERR_INVALID_ARG
    assert lib.lcsa_pipeline_create(C.byref(kv), 2, None, C.byref(h)) == _abi.ERR_INVALID_ARG
    assert h.value is None                                            # *out cleared on error
    assert lib.lcsa_pipeline_create(C.byref(kv), 0, C.byref(sp), C.byref(h)) == _abi.ERR_SHAPE
    assert lib.lcsa_pipeline_create(C.byref(kv), 8, C.byref(sp), C.byref(h)) == _abi.ERR_SHAPE   # > cap
    sp.window_mode = 7
    assert lib.lcsa_pipeline_create(C.byref(kv), 2, C.byref(sp), C.byref(h)) == _abi.ERR_INVALID_ARG
    sp.window_mode = 0
    kv.cap_frames = 5                                                 # odd capacity
    assert lib.lcsa_pipeline_create(C.byref(kv), 2, C.byref(sp), C.byref(h)) == _abi.ERR_SHAPE
    assert lib.lcsa_pipeline_submit(None, 0x1000, 0x1000, 0x1000, 0x1000) == _abi.ERR_INVALID_ARG
    assert lib.lcsa_pipeline_sync(None) == _abi.ERR_INVALID_ARG
    assert lib.lcsa_pipeline_start_timer(None) == _abi.ERR_INVALID_ARG
    ms = C.c_float()
    assert lib.lcsa_pipeline_elapsed_ms(None, C.byref(ms)) == _abi.ERR_INVALID_ARG
    lib.lcsa_pipeline_destroy(None)                                   # no-op


def test_select_kmax_host_rule(lib):
    from block_sparse_causal_lcsa_b200 import _abi
    kv = _abi.KVCacheStruct()
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 12, 6, 48, 88, 128
    kv.begin[0], kv.end[0] = 0, 6
    sp = _abi.SelectParamsStruct(0, 0, 0, 0, 0.136, 1e-5)
    assert lib.lcsa_select_kmax(C.byref(kv), 2, C.byref(sp)) == 27  # 198 candidates
    kv.Y, kv.X = 96, 168
    sp.window = 9
    assert lib.lcsa_select_kmax(C.byref(kv), 2, C.byref(sp)) == 34  # 243 candidates
    # workspace: 12 heads x 252 query blocks x 756 causal candidates x 8 bytes
    assert lib.lcsa_select_workspace_bytes(C.byref(kv), 2) == 12 * 252 * 756 * 8


def test_kv_advance_host_state(lib):
    """lcsa_kv_advance applies an append's cache-state update with no device
    work: first odd chunk, steady appends, eviction at the capacity."""
    from block_sparse_causal_lcsa_b200 import _abi
    kv = _abi.KVCacheStruct()
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 2, 1, 6, 16, 16, 128
    assert lib.lcsa_kv_advance(C.byref(kv), 3, 1, 0) == _abi.OK          # odd first chunk of stream 0
    assert (kv.begin[0], kv.end[0]) == (1, 4)
    assert lib.lcsa_kv_advance(C.byref(kv), 1, 1, 0) == _abi.ERR_SHAPE   # odd chunk on a non-empty stream
    for _ in range(3):
        assert lib.lcsa_kv_advance(C.byref(kv), 2, 2, 0) == _abi.OK
    assert (kv.begin[0], kv.end[0]) == (4, 10)                           # the newest 6 frames
    assert (kv.begin[1], kv.end[1]) == (0, 6)
    assert lib.lcsa_kv_advance(C.byref(kv), 2, 2, 1) == _abi.ERR_INVALID_ARG   # streams 1..2 of 2
    assert lib.lcsa_kv_advance(None, 2, 1, 0) == _abi.ERR_INVALID_ARG


def test_new_entry_points_reject_bad_arguments(lib):
    from block_sparse_causal_lcsa_b200 import _abi
    kv = _abi.KVCacheStruct()
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 1, 6, 16, 16, 128
    kv.begin[0], kv.end[0] = 0, 6
    t = _abi.Tensor(0x1000, 1, 1, 2, 16, 16, 128, 65536, 65536, 32768, 2048, 128)
    # token-window attention needs a token-level mode
    assert lib.lcsa_sparse_attn_fwd_window(C.byref(t), C.byref(kv), 0x5000, 0x6000, 4, 72, 0, C.byref(t), None,
                                           None) == _abi.ERR_INVALID_ARG
    assert lib.lcsa_sparse_attn_fwd_ex(C.byref(t), C.byref(kv), 0x5000, 0x6000, 4, -1, 2, C.byref(t), None, None, 0,
                                       None) == _abi.ERR_INVALID_ARG
    # window modes: token windows may be even, block windows may not; unknown modes are rejected
    sp = _abi.SelectParamsStruct(0, 72, 2, 64, 0.136, 1e-5)
    ws = lib.lcsa_select_workspace_bytes(C.byref(kv), 2)
    sp.window_mode = 4
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, ws, None) == \
        _abi.ERR_INVALID_ARG
    sp.window_mode = 1
    assert lib.lcsa_select_blocks(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000, 0x7000, ws, None) == \
        _abi.ERR_INVALID_ARG
    # segment lists: capacity below the longest segment's key blocks, segments longer than the queries
    assert lib.lcsa_segment_kmax(C.byref(kv)) == 3 * 4
    assert lib.lcsa_segment_blocks(6, C.byref(kv), 11, 0x5000, 0x6000, None) == _abi.ERR_CAPACITY
    assert lib.lcsa_segment_blocks(4, C.byref(kv), 12, 0x5000, 0x6000, None) == _abi.ERR_SHAPE
    # backward: workspace too small
    need = lib.lcsa_sparse_attn_bwd_workspace_bytes(C.byref(kv), 2)
    assert need > 0
    assert lib.lcsa_sparse_attn_bwd(C.byref(t), C.byref(kv), 0x5000, 0x6000, 4, C.byref(t), 0x8000, C.byref(t),
                                    C.byref(t), 0x9000, 0xA000, 0xB000, need - 16, None) == _abi.ERR_WORKSPACE
    assert lib.lcsa_sparse_attn_fwd_workspace_bytes(128) == 2 * 128 * 128 * 129 * 4
    assert lib.lcsa_sparse_attn_fwd_workspace_bytes(96) == 0


@pytest.mark.parametrize("mode,window", [(2, 72), (3, 72), (2, 20), (3, 35), (0, 9), (1, 9)])
def test_select_kmax_covers_every_row(lib, mode, window):
    """The host capacity rule bounds K_i of every row, token windows included
    (checked against the oracle's window and K rules)."""
    from block_sparse_causal_lcsa_b200 import _abi
    from oracle import lcsa_oracle as orc
    kv = _abi.KVCacheStruct()
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 1, 6, 96, 168, 128
    kv.begin[0], kv.end[0] = 0, 6
    sp = _abi.SelectParamsStruct(0, window, mode, 0, 0.136, 1e-5)
    kmax = lib.lcsa_select_kmax(C.byref(kv), 2, C.byref(sp))
    Hb, Wb = 12, 21
    Ks = []
    for i in range(Hb * Wb):
        yq, xq = divmod(i, Wb)
        C_i = int(orc.allowed_blocks(2, yq, xq, 3, Hb, Wb, window, mode).sum())
        Ks.append(orc.top_k_count(C_i, 0, 0.136))
    assert kmax >= max(Ks)
    assert kmax <= max(Ks) + 1 or mode >= 2


def test_binding_rejects_bad_selection_outputs(lib):
    """The Python binding checks dtype, shape, layout and device of q_pool and
    of caller-given blk_idx / blk_cnt before calling the library, so a wrong
    output can never be written past its end (ValueError, nothing launched)."""
    import torch
    import block_sparse_causal_lcsa_b200 as lc

    cache = lc.KVCache(1, 2, 6, 16, 24, 128, device="cpu")
    cache.struct.begin[0], cache.struct.end[0] = 0, 6
    params = lc.SelectParams(density=0.5)
    nQB, kmax = 1 * 2 * 3, 40
    good = dict(q_pool=torch.zeros((1, 2, 1, 2, 3, 128), dtype=torch.float64),
                blk_idx=torch.zeros((1, 2, nQB, kmax), dtype=torch.int32),
                blk_cnt=torch.zeros((1, 2, nQB), dtype=torch.int32))
    bad = [
        dict(blk_idx=good["blk_idx"].long()),                                    # int64 outputs
        dict(blk_cnt=good["blk_cnt"].long()),
        dict(blk_idx=torch.zeros((1, 2, nQB - 1, kmax), dtype=torch.int32)),     # too few rows
        dict(blk_cnt=torch.zeros((1, 2, nQB - 1), dtype=torch.int32)),
        dict(blk_idx=torch.zeros((1, 2, kmax, nQB), dtype=torch.int32).transpose(2, 3)),  # not contiguous
        dict(q_pool=good["q_pool"].float()),                                     # float32 pooled Q
        dict(q_pool=torch.zeros((1, 2, 2, 2, 3, 128), dtype=torch.float64)),     # q_pool of 2 time blocks
        dict(blk_idx=[0] * 10),                                                  # not a tensor
        {},                                                                      # right shapes, host memory
    ]
    for b in bad:
        a = {**good, **b}
        with pytest.raises(ValueError):
            lc.select_blocks_noalloc(a["q_pool"], 2, cache, params, a["blk_idx"], a["blk_cnt"])
        if isinstance(a["blk_idx"], torch.Tensor) and a["blk_idx"].dim() == 4:
            with pytest.raises(ValueError):
                lc.select_blocks(a["q_pool"], 2, cache, params, a["blk_idx"].shape[-1], a["blk_idx"],
                                 a["blk_cnt"], workspace=torch.zeros(16, dtype=torch.uint8))


def test_binding_rejects_bad_buffers_of_every_call(lib):
    """Every binding call that hands the library a bare pointer checks the
    buffer's dtype, shape and layout against what the call derives from its
    other arguments, then that all tensors sit on one GPU, before calling the
    library (ValueError naming the argument, nothing launched). On this host
    the all-good case stops at the device check."""
    import torch
    import block_sparse_causal_lcsa_b200 as lc

    bf, f32, f64, i32 = torch.bfloat16, torch.float32, torch.float64, torch.int32
    cache = lc.KVCache(1, 2, 6, 16, 24, 128, device="cpu")
    cache.struct.begin[0], cache.struct.end[0] = 0, 6
    q = torch.zeros((1, 2, 2, 16, 24, 128), dtype=bf)
    nQB, kmax = 1 * 2 * 3, 5
    idx, cnt = torch.zeros((1, 2, nQB, kmax), dtype=i32), torch.zeros((1, 2, nQB), dtype=i32)
    lse = torch.zeros((1, 2, 2, 16, 24), dtype=f32)
    ws = torch.zeros(64, dtype=torch.uint8)
    qp = torch.zeros((1, 2, 1, 2, 3, 128), dtype=f64)

    def fwd(**kw):
        a = dict(q=q, blk_idx=idx, blk_cnt=cnt, o=torch.empty_like(q), lse=lse, workspace=ws)
        a.update(kw)
        lc.sparse_attn_fwd(a["q"], cache, a["blk_idx"], a["blk_cnt"], a["o"], a["lse"], workspace=a["workspace"])

    cases = [
        (lambda: fwd(blk_idx=idx.long()), r"blk_idx must be torch\.int32"),
        (lambda: fwd(blk_idx=idx[0]), r"blk_idx must be an int32 tensor"),
        (lambda: fwd(blk_idx=idx[:, :, 1:]), r"blk_idx must have shape"),
        (lambda: fwd(blk_idx=torch.zeros((1, 2, kmax, nQB), dtype=i32).transpose(2, 3)), r"blk_idx must be contiguous"),
        (lambda: fwd(blk_cnt=cnt.long()), r"blk_cnt must be torch\.int32"),
        (lambda: fwd(blk_cnt=cnt[:, :, 1:]), r"blk_cnt must have shape"),
        (lambda: fwd(lse=lse.double()), r"lse must be torch\.float32"),
        (lambda: fwd(lse=lse[:, :, :1]), r"lse must have shape"),
        (lambda: fwd(o=torch.empty_like(q, dtype=f32)), r"o must be a bf16 tensor"),
        (lambda: fwd(q=q.float()), r"q must be a bf16 tensor"),
        (lambda: fwd(workspace=ws[::2]), r"workspace must be a contiguous"),
        (lambda: fwd(), r"q must be a CUDA tensor"),
        # backward: gradient buffers in the cache layout, the forward's LSE
        (lambda: lc.sparse_attn_bwd(q, cache, idx, cnt, q, lse, q, torch.empty_like(q),
                                    torch.zeros((1, 2, 4, 16, 24, 128), dtype=bf), torch.zeros_like(cache.v), ws),
         r"dk must have shape"),
        (lambda: lc.sparse_attn_bwd(q, cache, idx, cnt, q, lse, q, torch.empty_like(q), torch.zeros_like(cache.k),
                                    torch.zeros_like(cache.v, dtype=f32), ws), r"dv must be torch\.bfloat16"),
        (lambda: lc.sparse_attn_bwd(q, cache, idx, cnt, q, lse.half(), q, torch.empty_like(q),
                                    torch.zeros_like(cache.k), torch.zeros_like(cache.v), ws), r"lse must be torch\.float32"),
        (lambda: lc.sparse_attn_bwd(q, cache, idx, cnt, q, lse, q.float(), torch.empty_like(q),
                                    torch.zeros_like(cache.k), torch.zeros_like(cache.v), ws), r"d_o must be a bf16"),
        (lambda: lc.sparse_attn_bwd(q, cache, idx.long(), cnt, q, lse, q, torch.empty_like(q),
                                    torch.zeros_like(cache.k), torch.zeros_like(cache.v), ws), r"blk_idx must be torch\.int32"),
        (lambda: lc.sparse_attn_bwd(q, cache, idx, cnt, q, lse, q, torch.empty_like(q), torch.zeros_like(cache.k),
                                    torch.zeros_like(cache.v), ws), r"q must be a CUDA tensor"),
        # pooling, ingest and append: pooled rows [B,H,ceil(T/2),Y/8,X/8,D] in float64
        (lambda: lc.pool_qk(q, None, qp.float()), r"q_pool must be torch\.float64"),
        (lambda: lc.pool_qk(q, None, qp[:, :1]), r"q_pool must have shape"),
        (lambda: lc.pool_qk(q, q, qp, torch.zeros((1, 2, 2, 2, 3, 128), dtype=f64)), r"k_pool must have shape"),
        (lambda: lc.pool_qk(q, None, qp), r"q must be a CUDA tensor"),
        (lambda: lc.ingest_chunk(q, cache, q, q, torch.zeros((1, 2, 1, 2, 3, 64), dtype=f64)), r"q_pool must have shape"),
        (lambda: lc.ingest_chunk(q, cache, q, q.float(), qp), r"v_new must be a bf16"),
        (lambda: lc.ingest_chunk(q, cache, q, q, qp), r"cache must be a CUDA tensor"),
        (lambda: lc.kv_append(cache, q, q, qp.float()), r"k_pool_new must be torch\.float64"),
        (lambda: lc.kv_append(cache, q, q, torch.zeros((1, 2, 2, 2, 3, 128), dtype=f64)), r"k_pool_new must have shape"),
        (lambda: lc.kv_append(cache, q, q), r"cache must be a CUDA tensor"),
        # segment lists: kmax is blk_idx's last extent
        (lambda: lc.segment_blocks(2, cache, kmax + 1, idx, cnt), r"kmax 6 differs"),
        (lambda: lc.segment_blocks(2, cache, None, idx, cnt.long()), r"blk_cnt must be torch\.int32"),
        (lambda: lc.segment_blocks(2, cache, None, idx, cnt), r"cache must be a CUDA tensor"),
        # caller-given cache buffers
        (lambda: lc.KVCache(1, 2, 6, 16, 24, 128, device="cpu", k=torch.zeros((1, 2, 4, 16, 24, 128), dtype=bf)),
         r"k must have shape"),
        (lambda: lc.KVCache(1, 2, 6, 16, 24, 128, device="cpu",
                            k_pool=torch.zeros((1, 2, 3, 2, 3, 128), dtype=f32)), r"k_pool must be torch\.float64"),
        (lambda: lc.KVCache(1, 2, 6, 16, 24, 128, device="cpu",
                            v=torch.zeros((1, 2, 6, 16, 128, 24), dtype=bf).transpose(4, 5)), r"v must be contiguous"),
    ]
    for call, msg in cases:
        with pytest.raises(ValueError, match=msg):
            call()


def test_missing_or_incomplete_library_fails_loudly():
    """No silent fallback: a missing liblcsa.so, or a shared library without
    its entry points, raises ImportError at load."""
    import _ctypes
    from block_sparse_causal_lcsa_b200 import _abi
    with pytest.raises(ImportError, match="not built"):
        _abi.load("/nonexistent/liblcsa.so")
    with pytest.raises(ImportError, match="lacks the entry point lcsa_"):
        _abi.load(_ctypes.__file__)     # a real shared library with none of them
