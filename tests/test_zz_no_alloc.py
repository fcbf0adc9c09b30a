"""minikv_decode_attn_static: the decode step for callers that may not
allocate device memory (hosts whose device memory is all planned by their own
allocator, latency-critical loops where cudaMalloc may synchronize the
device).  It takes its scratch from a fixed array inside the library instead
of a caller workspace; its results must match minikv_decode_attn.

This file is named so that pytest collects it last.
"""
import ctypes
import math

import pytest
import torch

from bit_quantized_evicted_b200 import minikv as mk
from bit_quantized_evicted_b200 import synth

pytestmark = pytest.mark.gpu


def _run_steps(with_ws, no_alloc, B, Hq, Hkv, steps, dev):
    for step in range(steps):        # calls in a row share the static scratch
        q = synth.normal_fp16((B, Hq, 128), synth.seed_of(31, 0, synth.T_QDEC, step), dev)
        kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(31, 0, synth.T_KNEW, step), dev)
        vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(31, 0, synth.T_VNEW, step), dev)
        ref = mk.decode_attn(with_ws, q, kn, vn)
        got = mk.decode_attn_static(no_alloc, q, kn, vn)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (step, float((got.float() - ref.float()).abs().max()))
        assert (no_alloc.n_packed, no_alloc.n_res, no_alloc.res_start) == \
            (with_ws.n_packed, with_ws.n_res, with_ws.res_start)


@pytest.mark.gpu
def test_static_scratch_decode_matches_workspace_decode_twice():
    """Both entry points run the same kernel on the same plan; with the fixed
    item-to-warp assignment (minikv_set_deterministic) their outputs must be
    bit-identical, step after step.  From N = 1000 kept tokens
    (R = 128, G = 32) the residual starts at 136 tokens and reaches R + G = 160
    at step 24, so the run also flushes a key group through the static
    scratch; the packed caches must then be identical too."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = "cuda"
    B, Hq, Hkv, N, R, G, steps = 2, 8, 2, 1000, 128, 32, 27
    k = synth.keys_fp16((B, Hkv, N, 128), synth.seed_of(31, 0, synth.T_K), dev)
    v = synth.normal_fp16((B, Hkv, N, 128), synth.seed_of(31, 0, synth.T_V), dev)
    cap = ((N + steps) // G + 2) * G
    with_ws = mk.MiniKVCache(B, Hkv, cap, R=R, G=G, Hq=Hq, device=dev)
    no_alloc = mk.MiniKVCache(B, Hkv, cap, R=R, G=G, Hq=Hq, device=dev)
    mk.quant_pack(with_ws, k, v)
    mk.quant_pack(no_alloc, k, v)
    n_packed0 = with_ws.n_packed
    mk.set_deterministic(True)
    try:
        _run_steps(with_ws, no_alloc, B, Hq, Hkv, steps, dev)
    finally:
        mk.set_deterministic(False)
    assert with_ws.n_packed == n_packed0 + G     # one key group was flushed
    a, b = with_ws.arrays(), no_alloc.arrays()
    for name in a:
        assert torch.equal(a[name], b[name]), name


@pytest.mark.gpu
def test_static_scratch_rejects_a_step_above_its_size():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = mk.lib()
    c = mk.CacheStruct()
    B, Hkv, cap = 512, 8, 64
    n = L.minikv_cache_bytes(B, Hkv, 128, 32, 128, 32, cap)
    assert L.minikv_cache_bind(ctypes.byref(c), 1 << 24, n, B, Hkv, 128, 32, 128, 32, cap) == 0
    c.n_packed, c.n_res = 64, 32     # 4096 (sequence, KV head) units x 2 splits: above 8 MiB
    p = 1 << 30
    rc = L.minikv_decode_attn_static(ctypes.byref(c), p, p, p, 2 * Hkv, 1.0 / math.sqrt(128), p, None)
    assert rc == mk.ERR_UNSUPPORTED
    assert b"static buffer" in L.minikv_last_error_string()
    assert (c.n_packed, c.n_res) == (64, 32)
