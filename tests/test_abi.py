"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, carves a cache, and rejects bad arguments with the documented codes
before touching the device."""
import ctypes
import re

import pytest

from bit_quantized_evicted_b200 import minikv as mk


def _header_symbols():
    text = open(mk.HEADER_PATH).read()
    return sorted(set(re.findall(r"MINIKV_API\s+[\w\s\*]*?\b(minikv_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    syms = _header_symbols()
    for name in ("minikv_quant_pack", "minikv_select_prefill", "minikv_topk_evict", "minikv_decode_attn",
                 "minikv_workspace_size", "minikv_last_error_string"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    L = mk.lib()
    for name in _header_symbols():
        assert hasattr(L, name), name


def test_cache_bytes_and_bind():
    L = mk.lib()
    n = L.minikv_cache_bytes(16, 8, 128, 32, 128, 128, 6656)
    # codes 2 x 16*8*6656*32 B = 2 x 27262976, k scale/zero 2 x 128*208*256 B, v scale/zero 2 x 128*6656*2 B, ring 2 x 128*160*256 B
    assert n == 2 * 27262976 + 2 * 6815744 + 2 * 1703936 + 2 * 5242880
    c = mk.CacheStruct()
    base = 1 << 20    # never dereferenced: bind only does arithmetic
    assert L.minikv_cache_bind(ctypes.byref(c), base, n, 16, 8, 128, 32, 128, 128, 6656) == 0
    assert c.k_codes == base and c.v_codes == base + 27262976
    assert (c.n_packed, c.n_res, c.res_start) == (0, 0, 0)
    assert L.minikv_cache_bind(ctypes.byref(c), base, n - 1, 16, 8, 128, 32, 128, 128, 6656) == mk.ERR_INVALID_ARG


@pytest.mark.parametrize("shape,code", [
    ((1, 1, 64, 32, 128, 32, 64), mk.ERR_UNSUPPORTED),     # D != 128
    ((1, 1, 128, 48, 128, 32, 96), mk.ERR_UNSUPPORTED),    # G not a multiple of 32
    ((1, 1, 128, 32, 100, 32, 64), mk.ERR_UNSUPPORTED),    # Gv not a power of two <= 128
    ((1, 1, 128, 32, 128, 32, 50), mk.ERR_INVALID_ARG),    # cap not a multiple of G
    ((0, 1, 128, 32, 128, 32, 64), mk.ERR_INVALID_ARG),
])
def test_cache_shape_errors(shape, code):
    L = mk.lib()
    assert L.minikv_cache_bytes(*shape) == 0
    c = mk.CacheStruct()
    assert L.minikv_cache_bind(ctypes.byref(c), 1 << 20, 1 << 30, *shape) == code
    assert L.minikv_last_error_string()


def _bound_cache(B=1, Hkv=2, G=32, Gv=128, R=32, cap=256):
    L = mk.lib()
    c = mk.CacheStruct()
    n = L.minikv_cache_bytes(B, Hkv, 128, G, Gv, R, cap)
    assert L.minikv_cache_bind(ctypes.byref(c), 1 << 20, n, B, Hkv, 128, G, Gv, R, cap) == 0
    return c


def test_decode_argument_errors_before_any_launch():
    L = mk.lib()
    c = _bound_cache()
    p = 1 << 24
    # Hq not a multiple of Hkv
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 3, 0.1, p, p, 1 << 20, None) == mk.ERR_INVALID_ARG
    # more than 4 query heads per KV head
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 10, 0.1, p, p, 1 << 20, None) == mk.ERR_UNSUPPORTED
    # null output
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 2, 0.1, None, p, 1 << 20, None) == mk.ERR_INVALID_ARG
    # misaligned query
    assert L.minikv_decode_attn(ctypes.byref(c), p + 2, p, p, 2, 0.1, p, p, 1 << 20, None) == mk.ERR_INVALID_ARG
    # capacity: the cache is full and this step would flush a group
    c.n_packed, c.n_res = c.cap, c.R + c.G - 1
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 2, 0.1, p, p, 1 << 20, None) == mk.ERR_CAPACITY
    assert b"cap" in L.minikv_last_error_string()
    assert (c.n_packed, c.n_res) == (c.cap, c.R + c.G - 1)    # unchanged on error
    # inconsistent state
    c.n_packed = 17
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 2, 0.1, p, p, 1 << 20, None) == mk.ERR_INVALID_ARG


def test_pack_argument_errors():
    L = mk.lib()
    c = _bound_cache(cap=64)
    p = 1 << 24
    assert L.minikv_quant_pack(ctypes.byref(c), p, p, -1, None) == mk.ERR_INVALID_ARG
    assert L.minikv_quant_pack(ctypes.byref(c), None, p, 10, None) == mk.ERR_INVALID_ARG
    # 300 tokens, R=32, G=32 -> 256 packed > cap 64
    assert L.minikv_quant_pack(ctypes.byref(c), p, p, 300, None) == mk.ERR_CAPACITY
    assert L.minikv_quant_pack(None, p, p, 10, None) == mk.ERR_INVALID_ARG


def test_prefill_and_topk_argument_errors():
    L = mk.lib()
    p = 1 << 24
    ws = 1 << 20
    ok = (p, p, p, 1, 4, 4, 512, 128, 32, 0.088, p, p, p, ws, None)
    bad_w = (p, p, p, 1, 4, 4, 512, 128, 513, 0.088, p, p, p, ws, None)
    bad_d = (p, p, p, 1, 4, 4, 512, 64, 32, 0.088, p, p, p, ws, None)
    bad_h = (p, p, p, 1, 6, 4, 512, 128, 32, 0.088, p, p, p, ws, None)
    small_ws = (p, p, p, 1, 4, 4, 512, 128, 32, 0.088, p, p, p, 16, None)
    assert L.minikv_select_prefill(*bad_w) == mk.ERR_INVALID_ARG
    assert L.minikv_select_prefill(*bad_d) == mk.ERR_UNSUPPORTED
    assert L.minikv_select_prefill(*bad_h) == mk.ERR_INVALID_ARG
    assert L.minikv_select_prefill(*small_ws) == mk.ERR_INVALID_ARG
    assert len(ok) == 15
    # window above the budget
    assert L.minikv_topk_evict(p, p, p, 1, 4, 512, 128, 64, 32, p, p, p, None, 0, None) == mk.ERR_INVALID_ARG
    assert L.minikv_topk_evict(p, p, p, 1, 4, 512, 128, 32, 0, p, p, p, None, 0, None) == mk.ERR_INVALID_ARG
    assert L.minikv_topk_evict(p, p, p, 1, 4, 512, 96, 32, 64, p, p, p, None, 0, None) == mk.ERR_UNSUPPORTED


def test_select_prefill_status_argument_errors():
    L = mk.lib()
    st = ctypes.c_uint(0)
    p = ctypes.c_void_p(1 << 20)
    assert L.minikv_select_prefill_status(None, 4352, 1, 32, 32, None, ctypes.byref(st)) == mk.ERR_INVALID_ARG
    assert L.minikv_select_prefill_status(p, 4352, 1, 32, 32, None, None) == mk.ERR_INVALID_ARG
    assert L.minikv_select_prefill_status(p, 4351, 1, 32, 32, None, ctypes.byref(st)) == mk.ERR_INVALID_ARG
    assert L.minikv_select_prefill_status(p, 4352, 0, 32, 32, None, ctypes.byref(st)) == mk.ERR_INVALID_ARG


def test_workspace_sizes():
    # window rows' log-sum-exp (32 heads x 32 rows x 4 B), then the 256-byte status block
    assert mk.workspace_size(mk.OP_SELECT_PREFILL, 1, 32, 32, 4096, 128, 32) == 4096 + 256
    assert mk.workspace_size(mk.OP_TOPK_EVICT, 1, 32, 32, 4096, 128, 32) == 0
    assert mk.workspace_size(mk.OP_DECODE_ATTN, 16, 32, 8, 6656 + 160, 128) > 16 * 8 * 4


def test_evict_pack_argument_errors():
    L = mk.lib()
    c = _bound_cache(B=1, Hkv=2, cap=64)
    p = 1 << 24
    # B / Hkv must match the cache
    assert L.minikv_evict_pack(p, p, p, 1, 3, 512, 128, 32, 96, p, ctypes.byref(c), None) == mk.ERR_INVALID_ARG
    # window above the budget; empty budget; null index list
    assert L.minikv_evict_pack(p, p, p, 1, 2, 512, 128, 64, 32, p, ctypes.byref(c), None) == mk.ERR_INVALID_ARG
    assert L.minikv_evict_pack(p, p, p, 1, 2, 512, 128, 32, 0, p, ctypes.byref(c), None) == mk.ERR_INVALID_ARG
    assert L.minikv_evict_pack(p, p, p, 1, 2, 512, 128, 32, 96, None, ctypes.byref(c), None) == mk.ERR_INVALID_ARG
    # D != 128
    assert L.minikv_evict_pack(p, p, p, 1, 2, 512, 96, 32, 96, p, ctypes.byref(c), None) == mk.ERR_UNSUPPORTED
    # keep 300 of 512 with R=32, G=32 -> 256 packed > cap 64
    assert L.minikv_evict_pack(p, p, p, 1, 2, 512, 128, 32, 300, p, ctypes.byref(c), None) == mk.ERR_CAPACITY
    assert b"cap" in L.minikv_last_error_string()
    # misaligned K
    assert L.minikv_evict_pack(p, p + 2, p, 1, 2, 512, 128, 32, 96, p, ctypes.byref(c), None) == mk.ERR_INVALID_ARG
    assert (c.n_packed, c.n_res, c.res_start) == (0, 0, 0)   # the cache state is untouched on error


def test_ragged_cache_state_and_argument_errors():
    """Per-sequence host state: set_ragged resets it, the loaders reject a
    non-ragged cache or a bad row, and a bad per-sequence state is refused
    before any launch."""
    L = mk.lib()
    p = 1 << 24
    c = _bound_cache(B=3, Hkv=2, cap=256)
    assert c.seq is None
    # loaders of one sequence need a ragged cache
    assert L.minikv_quant_pack_seq(ctypes.byref(c), 0, p, p, 10, None) == mk.ERR_INVALID_ARG
    assert L.minikv_evict_pack_seq(p, p, p, 2, 512, 128, 32, 96, p, ctypes.byref(c), 0, None) == mk.ERR_INVALID_ARG
    seq = (ctypes.c_int * 9)(*range(1, 10))
    assert L.minikv_cache_set_ragged(ctypes.byref(c), ctypes.cast(seq, ctypes.c_void_p)) == 0
    assert list(seq) == [0] * 9
    assert c.seq is not None
    # row outside [0, B); capacity of one row; Hkv mismatch; negative row
    assert L.minikv_quant_pack_seq(ctypes.byref(c), 3, p, p, 10, None) == mk.ERR_INVALID_ARG
    assert L.minikv_quant_pack_seq(ctypes.byref(c), -1, p, p, 10, None) == mk.ERR_INVALID_ARG
    assert L.minikv_quant_pack_seq(ctypes.byref(c), 1, p, p, 400, None) == mk.ERR_CAPACITY
    assert L.minikv_evict_pack_seq(p, p, p, 3, 512, 128, 32, 96, p, ctypes.byref(c), 0, None) == mk.ERR_INVALID_ARG
    assert L.minikv_evict_pack_seq(p, p, p, 2, 512, 128, 32, 96, p, ctypes.byref(c), -2, None) == mk.ERR_INVALID_ARG
    assert L.minikv_evict_pack_seq(p, p, p, 2, 512, 128, 32, 330, p, ctypes.byref(c), 2, None) == mk.ERR_CAPACITY
    assert list(seq) == [0] * 9
    # an inconsistent state of one sequence, and a flush past capacity in one sequence
    seq[3 * 1] = 17
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 2, 0.1, p, p, 1 << 20, None) == mk.ERR_INVALID_ARG
    assert b"sequence 1" in L.minikv_last_error_string()
    seq[3 * 1] = 0
    seq[3 * 2], seq[3 * 2 + 1] = 256, 32 + 32 - 1
    assert L.minikv_decode_attn(ctypes.byref(c), p, p, p, 2, 0.1, p, p, 1 << 20, None) == mk.ERR_CAPACITY
    assert b"sequence 2" in L.minikv_last_error_string()
    assert (seq[6], seq[7]) == (256, 63)
    # back to a uniform batch
    assert L.minikv_cache_set_ragged(ctypes.byref(c), None) == 0
    assert c.seq is None and (c.n_packed, c.n_res, c.res_start) == (0, 0, 0)


def test_ragged_batch_limit():
    L = mk.lib()
    c = _bound_cache(B=mk.MAX_RAGGED_SEQS + 1, Hkv=1, cap=64)
    seq = (ctypes.c_int * (3 * (mk.MAX_RAGGED_SEQS + 1)))()
    assert L.minikv_cache_set_ragged(ctypes.byref(c), ctypes.cast(seq, ctypes.c_void_p)) == mk.ERR_UNSUPPORTED
    assert c.seq is None


def test_set_deterministic_is_a_host_switch():
    """The schedule switch needs no device: it only sets what the next decode
    call passes to its kernel."""
    L = mk.lib()
    assert L.minikv_set_deterministic(1) == 0
    assert L.minikv_set_deterministic(0) == 0
