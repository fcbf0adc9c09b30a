"""Failure reporting of the flash-attention pass, without a GPU fault.

Every wait of the tcgen05 pipeline in minikv_select_prefill is bounded; when
one gives up, the CTA waits for the copies and tensor-core operations it had
started, skips its outputs and sets bit 0 of the call's status word.  The
probe build of the library (same sources, waits cut to one poll) makes those
waits run out while their copies are really in flight; the test checks that
the call returns, the status reports the expiry, and the context still runs
the normal library correctly afterwards.
"""
import ctypes
import math
import os

import numpy as np
import pytest
import torch

from bit_quantized_evicted_b200 import build as B
from bit_quantized_evicted_b200 import minikv as mk
from bit_quantized_evicted_b200 import synth
from oracle import minikv_oracle as O

pytestmark = pytest.mark.gpu

_P, _I, _F, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t


def _probe():
    if not os.path.exists(B.WAIT_PROBE_LIB):
        pytest.fail(f"{B.WAIT_PROBE_LIB} is missing: build the library first")
    L = ctypes.CDLL(B.WAIT_PROBE_LIB)
    L.minikv_select_prefill.restype = _I
    L.minikv_select_prefill.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _Z, _P]
    L.minikv_select_prefill_status.restype = _I
    L.minikv_select_prefill_status.argtypes = [_P, _Z, _I, _I, _I, _P, ctypes.POINTER(ctypes.c_uint)]
    L.minikv_workspace_size.restype = _Z
    L.minikv_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I, _I]
    return L


def test_expired_waits_set_the_status_and_leave_the_context_usable():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mk.lib()
    dev = "cuda"
    Bn, H, T, W = 1, 2, 384, 32
    tau = 1.0 / math.sqrt(128.0)
    q = synth.normal_fp16((Bn, H, T, 128), synth.seed_of(201, 0, synth.T_Q), dev)
    k = synth.keys_fp16((Bn, H, T, 128), synth.seed_of(201, 0, synth.T_K), dev)
    v = synth.normal_fp16((Bn, H, T, 128), synth.seed_of(201, 0, synth.T_V), dev)
    o = torch.empty_like(q)
    sc = torch.empty((Bn, H, T), dtype=torch.float32, device=dev)
    probe = _probe()
    need = probe.minikv_workspace_size(mk.OP_SELECT_PREFILL, Bn, H, H, T, 128, W)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):   # two calls in a row: each clears the word and sets it again
        rc = probe.minikv_select_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), Bn, H, H, T, 128, W, tau,
                                         o.data_ptr(), sc.data_ptr(), ws.data_ptr(), ws.numel(), stream)
        assert rc == mk.OK
        st = ctypes.c_uint(7)
        assert probe.minikv_select_prefill_status(ws.data_ptr(), ws.numel(), Bn, H, W, stream, ctypes.byref(st)) == 0
        assert st.value == 1, st.value
    torch.cuda.synchronize()   # the kernels returned: nothing hung, nothing faulted
    # the same context, the normal library: the status reads 0 and the results are right
    o2, sc2 = mk.select_prefill(q, k, v, W, ws=ws)
    assert mk.select_prefill_status(ws, Bn, H, W) == 0
    on = o2.float().cpu().numpy()
    for h in range(H):
        ref = O.prefill_attention(q[0, h].cpu().numpy(), k[0, h].cpu().numpy(), v[0, h].cpu().numpy(), tau)
        assert float(np.max(np.abs(on[0, h] - ref))) <= 2e-3
