"""Host logic of the decode partition (minikv_decode_plan), on CPU.

The decode work list holds, for each (sequence, KV head) unit in order,
ceil((n_res + 1) / 5) residual items and then n_packed / 32 packed items; the
host cuts it into one contiguous range per CTA at a boundary weight it picks
per call from a cost model of the slowest CTA.  These tests check the cut's
invariants on many states, and the weight the model picks for the batch
shapes it was fitted on (the Mistral-7B GQA decode batch gets one CTA per
unit, the ragged and LLaMA2-13B batches a small weight).  Without a GPU the
library assumes 148 SMs.
"""
import ctypes
import threading

import numpy as np
import pytest

from bit_quantized_evicted_b200 import minikv as mk
from oracle import minikv_oracle as O

CANDIDATES = {128, 256, 512, 896, 1280, 1 << 20}
SMS = 148


def _bound(B, Hkv, cap, G=32, R=128):
    L = mk.lib()
    c = mk.CacheStruct()
    n = L.minikv_cache_bytes(B, Hkv, 128, G, 128, R, cap)
    assert n > 0
    assert L.minikv_cache_bind(ctypes.byref(c), 1 << 20, n, B, Hkv, 128, G, 128, R, cap) == 0
    return c


def _items(n_packed, n_res):
    return -(-(n_res + 1) // 5) + n_packed // 32


def _ragged(c, states):
    seq = (ctypes.c_int * (3 * len(states)))()
    assert mk.lib().minikv_cache_set_ragged(ctypes.byref(c), ctypes.cast(seq, ctypes.c_void_p)) == 0
    for b, (nq, nr) in enumerate(states):   # set_ragged empties the table; then each row's state
        seq[3 * b], seq[3 * b + 1], seq[3 * b + 2] = nq, nr, 0
    return seq   # keep the host table alive


def _check_cut(ctas, wu, first, unit_items):
    assert 1 <= ctas <= SMS
    assert wu in CANDIDATES
    assert len(first) == ctas + 1
    assert first[0] == 0 and first[-1] == sum(unit_items)
    assert all(a < b for a, b in zip(first, first[1:])), "every CTA gets at least one item"


def test_mistral_gqa_batch_gets_one_cta_per_unit():
    """B=16, Hkv=8, 20 % of 32K kept (6400 packed + 153 residual tokens): 128
    units of 231 items, a little larger than a 148-way share; the model keeps
    each unit whole."""
    nq, nr = O.split(32768 * 20 // 100, 128, 32)
    c = _bound(16, 8, 6656)
    c.n_packed, c.n_res = nq, nr
    ctas, wu, first = mk.decode_plan(c)
    assert (ctas, wu) == (128, 1 << 20)
    assert first == [231 * i for i in range(129)]


def test_llama2_13b_batch_splits_units_at_a_small_weight():
    nq, nr = O.split(16384 * 15 // 100, 128, 32)
    c = _bound(8, 40, nq + 160)
    c.n_packed, c.n_res = nq, nr
    ctas, wu, first = mk.decode_plan(c)
    assert (ctas, wu) == (148, 128)
    _check_cut(ctas, wu, first, [_items(nq, nr)] * 320)


def test_ragged_batch_splits_units_at_a_small_weight():
    states = [O.split((4096 + (32768 - 4096) * b // 15) * 20 // 100, 128, 32) for b in range(16)]
    c = _bound(16, 8, 6656)
    keep = _ragged(c, states)
    ctas, wu, first = mk.decode_plan(c)
    assert (ctas, wu) == (148, 256)
    _check_cut(ctas, wu, first, [_items(nq, nr) for nq, nr in states for _ in range(8)])
    del keep


@pytest.mark.parametrize("seed", range(12))
def test_cut_invariants_on_random_states(seed):
    rng = np.random.default_rng(seed)
    B, Hkv = int(rng.integers(1, 33)), int(rng.choice([1, 2, 4, 8, 32, 40]))
    cap = 32 * int(rng.integers(1, 400))
    c = _bound(B, Hkv, cap)
    if rng.random() < 0.5:
        nq, nr = 32 * int(rng.integers(0, cap // 32 + 1)), int(rng.integers(0, 160))
        c.n_packed, c.n_res = nq, nr
        units = [_items(nq, nr)] * (B * Hkv)
        keep = None
    else:
        states = [(32 * int(rng.integers(0, cap // 32 + 1)), int(rng.integers(0, 160))) for _ in range(B)]
        keep = _ragged(c, states)
        units = [_items(nq, nr) for nq, nr in states for _ in range(Hkv)]
    ctas, wu, first = mk.decode_plan(c)
    _check_cut(ctas, wu, first, units)
    assert mk.decode_plan(c) == (ctas, wu, first), "the same state always gets the same cut"
    out = []
    t = threading.Thread(target=lambda: out.append(mk.decode_plan(c)))
    t.start()
    t.join()
    assert out == [(ctas, wu, first)], "and so does another host thread"
    del keep


def test_first_items_buffer_too_small_is_rejected():
    c = _bound(4, 8, 640)
    c.n_packed, c.n_res = 320, 100
    ctas, wu, _ = mk.decode_plan(c)
    buf = (ctypes.c_int * ctas)()
    n, w = ctypes.c_int(0), ctypes.c_int(0)
    rc = mk.lib().minikv_decode_plan(ctypes.byref(c), ctypes.byref(n), ctypes.byref(w), buf, ctas)
    assert rc == mk.ERR_INVALID_ARG
    assert rc == mk.lib().minikv_decode_plan(None, ctypes.byref(n), ctypes.byref(w), None, 0)
