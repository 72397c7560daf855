"""lcsa_select_blocks_noalloc: block selection with the library's own fixed
scratch array instead of a workspace from the caller.

It serves callers that cannot allocate device memory: a plugin or engine
whose device memory all belongs to a host framework's pool, or a real-time
frame loop that must not call cudaMalloc because an allocation can
synchronise the device and stall the stream. Its selections must equal those
of lcsa_select_blocks bit for bit, including on consecutive calls, which
share the scratch array and find the previous call's contents in it.

This file is collected last, so it runs both after every other test and,
alone, in a fresh process.
"""
import ctypes as C
import os

import pytest
import torch

import lcsa_inputs as li

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    import importlib.util

    # load build.py by path: importing the package first would load a stale library
    spec = importlib.util.spec_from_file_location(
        "lcsa_build", os.path.join(ROOT, "block_sparse_causal_lcsa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    from block_sparse_causal_lcsa_b200 import _abi
    return _abi, _abi.load()


def test_oversized_request_rejected_before_device_work():
    """A selection that needs more scratch than the fixed array holds (one
    1536x2688 stream: 12 heads x 252 query blocks x 756 candidates x 8 bytes)
    is refused with its own status, before any CUDA call (no GPU here)."""
    _abi, lib = _lib()
    kv = _abi.KVCacheStruct()
    kv.k, kv.v, kv.k_pool = 0x1000, 0x2000, 0x3000
    kv.B, kv.H, kv.cap_frames, kv.Y, kv.X, kv.D = 1, 12, 6, 96, 168, 128
    kv.begin[0], kv.end[0] = 0, 6
    sp = _abi.SelectParamsStruct(0, 9, 0, 64, 0.136, 1e-5)
    assert lib.lcsa_select_workspace_bytes(C.byref(kv), 2) > _abi.SELECT_STATIC_SCRATCH_BYTES
    assert lib.lcsa_select_blocks_noalloc(0x4000, 2, C.byref(kv), C.byref(sp), 0x5000, 0x6000,
                                          None) == _abi.ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.lcsa_status_string(_abi.ERR_SCRATCH_LIMIT)


@pytest.mark.gpu
def test_noalloc_matches_workspace_select_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    _abi, lib = _lib()
    import block_sparse_causal_lcsa_b200 as lc
    from lcsa_harness import build_cache, params_of

    # four 768x1408 streams (6.7 MB of scratch), then one (1.3 MB): the second
    # call finds the first call's keys in the shared array
    cases = []
    for w in (li.workload("multistream"), li.workload("chunk")):
        x = li.make_inputs(w)
        cache, k_new, v_new = build_cache(lc, w, x, "cuda")
        lc.kv_append(cache, k_new, v_new, lc.pool_qk(k_new)[0])
        q_pool = lc.pool_qk(x["q"].to("cuda"))[0]
        params = params_of(lc, w)
        assert 0 < lc.select_workspace_bytes(cache, w.q_frames) <= _abi.SELECT_STATIC_SCRATCH_BYTES
        ref_idx, ref_cnt = lc.select_blocks(q_pool, w.q_frames, cache, params)
        cases.append((w, cache, q_pool, params, ref_idx, ref_cnt))
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0

    outs = []
    for w, cache, q_pool, params, ref_idx, ref_cnt in cases:
        idx = torch.full_like(ref_idx, 7777)  # every entry must be written
        cnt = torch.full_like(ref_cnt, 7777)
        sp = params.struct(ref_idx.shape[-1])
        st = lib.lcsa_select_blocks_noalloc(q_pool.data_ptr(), w.q_frames, C.byref(cache.struct),
                                            C.byref(sp), idx.data_ptr(), cnt.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
        assert st == _abi.OK, lib.lcsa_status_string(st)
        outs.append((idx, cnt))
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    for (w, _, _, _, ref_idx, ref_cnt), (idx, cnt) in zip(cases, outs):
        assert torch.equal(cnt, ref_cnt), w.name
        assert torch.equal(idx, ref_idx), w.name

    # and once more through the Python binding, which checks the outputs'
    # dtype, shape and device before the same C call
    w, cache, q_pool, params, ref_idx, ref_cnt = cases[0]
    idx = torch.full_like(ref_idx, 7777)
    cnt = torch.full_like(ref_cnt, 7777)
    lc.select_blocks_noalloc(q_pool, w.q_frames, cache, params, idx, cnt)
    torch.cuda.synchronize()
    assert lc.last_device_error() == 0
    assert torch.equal(cnt, ref_cnt) and torch.equal(idx, ref_idx)
