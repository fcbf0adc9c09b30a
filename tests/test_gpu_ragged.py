"""Ragged batches (each sequence with its own packed and residual lengths)
through the C ABI, against the CPU oracle.

The oracle keeps one slice per (sequence, KV head) anyway, so a ragged batch is
a list of slices built from prompts of different lengths.  Bars as for uniform
batches: codes, scales, zeros and residual rows bit-exact; outputs within 2e-3
max-abs of the fp64 oracle; running attention masses within 2e-5 per step.
"""
import math

import numpy as np
import pytest
import torch

from bit_quantized_evicted_b200 import minikv as mk
from bit_quantized_evicted_b200 import synth
from oracle import minikv_oracle as O
from tests.oracle_runs import np16

pytestmark = pytest.mark.gpu

ATOL_OUT = 2e-3
ATOL_MASS_PER_STEP = 2e-5
TAU = 1.0 / math.sqrt(128.0)
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mk.lib()


def _seq_kv(Hkv, N, seed):
    k = synth.keys_fp16((Hkv, N, 128), synth.seed_of(seed, N, synth.T_K), DEV)
    v = synth.normal_fp16((Hkv, N, 128), synth.seed_of(seed, N, synth.T_V), DEV)
    return k, v


def _load(lengths, Hq, Hkv, G, R, steps, seed, device_state=False, cap=None):
    """A ragged cache (host-side or device-resident per-sequence state) loaded
    sequence by sequence, and the oracle's slices."""
    B = len(lengths)
    if cap is None:
        cap = ((max(lengths) + steps) // G + 2) * G
    cache = mk.MiniKVCache(B, Hkv, cap, G=G, Gv=128, R=R, Hq=Hq)
    cache.set_device_state() if device_state else cache.set_ragged()
    ref = []
    for b, N in enumerate(lengths):
        k, v = _seq_kv(Hkv, N, seed + b)
        mk.quant_pack_seq(cache, b, k, v)
        kn, vn = np16(k), np16(v)
        ref.append([O.SliceCache.from_kept(kn[h], vn[h], R, G, 128) for h in range(Hkv)])
    return cache, ref


def _step_inputs(B, Hq, Hkv, seed, s):
    q = synth.normal_fp16((B, Hq, 128), synth.seed_of(seed, 0, synth.T_QDEC, s), DEV)
    kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(seed, 0, synth.T_KNEW, s), DEV)
    vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(seed, 0, synth.T_VNEW, s), DEV)
    return q, kn, vn


def _compare_seq(cache, b, slices):
    """Sequence b of the GPU cache against the oracle slices, bit for bit."""
    a = {k: v.cpu().numpy() for k, v in cache.arrays().items()}
    kr, vr = (t.cpu().numpy() for t in cache.residual_seq(b))
    G = cache.G
    for h, s in enumerate(slices):
        nq = s.n_q
        assert cache.seq_state(b)[:2] == (nq, s.r), (b, cache.seq_state(b), nq, s.r)
        np.testing.assert_array_equal(a["k_codes"][b, h, :nq].view(np.uint32), s.k_codes)
        np.testing.assert_array_equal(a["v_codes"][b, h, :nq].view(np.uint32), s.v_codes)
        np.testing.assert_array_equal(a["k_scale"][b, h, :nq // G].view(np.uint16), s.k_scale)
        np.testing.assert_array_equal(a["k_zero"][b, h, :nq // G].view(np.uint16), s.k_zero)
        np.testing.assert_array_equal(a["v_scale"][b, h, :nq].view(np.uint16), s.v_scale)
        np.testing.assert_array_equal(a["v_zero"][b, h, :nq].view(np.uint16), s.v_zero)
        np.testing.assert_array_equal(kr[h].view(np.uint16), np.array(s.res_k, np.uint16).reshape(s.r, 128))
        np.testing.assert_array_equal(vr[h].view(np.uint16), np.array(s.res_v, np.uint16).reshape(s.r, 128))


@pytest.mark.parametrize("device_state", [False, True])
@pytest.mark.parametrize("lengths,Hq,Hkv,G,R,steps", [
    ((300, 20, 1000, 0, 161), 8, 2, 32, 32, 40),        # g = 4; an empty and an all-residual sequence
    ((700, 64, 2100), 4, 4, 64, 64, 70),                # g = 1, G = 64, flushes at different steps
    ((96, 33, 129, 500, 1, 64), 3, 1, 32, 0, 35),       # g = 3, R = 0
])
def test_ragged_decode_vs_oracle(lengths, Hq, Hkv, G, R, steps, device_state):
    B = len(lengths)
    g = Hq // Hkv
    cache, ref = _load(lengths, Hq, Hkv, G, R, steps, 700, device_state)
    for b in range(B):
        _compare_seq(cache, b, ref[b])
    worst = 0.0
    for s in range(steps):
        q, kn, vn = _step_inputs(B, Hq, Hkv, 71, s)
        out = mk.decode_attn(cache, q, kn, vn)
        torch.cuda.synchronize()
        qn, knn, vnn = np16(q), np16(kn), np16(vn)
        got = out.float().cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                o = ref[b][h].step(qn[b, h * g:(h + 1) * g], knn[b, h], vnn[b, h], TAU)
                err = float(np.max(np.abs(got[b, h * g:(h + 1) * g] - o)))
                worst = max(worst, err)
                assert err <= ATOL_OUT, (s, b, h, err)
    for b in range(B):
        _compare_seq(cache, b, ref[b])
    print(f"ragged decode max-abs error {worst:.2e}")


@pytest.fixture
def deterministic():
    mk.set_deterministic(True)
    try:
        yield
    finally:
        mk.set_deterministic(False)


def test_ragged_equal_lengths_match_uniform_bit_for_bit(deterministic):
    """A ragged batch whose sequences all have the same length runs the same
    schedule as the uniform batch: identical outputs and cache bytes (with the
    fixed item-to-warp assignment; dynamic claiming may round differently)."""
    B, Hq, Hkv, N, steps = 4, 8, 2, 1000, 3
    k = synth.keys_fp16((B, Hkv, N, 128), synth.seed_of(77, 0, synth.T_K), DEV)
    v = synth.normal_fp16((B, Hkv, N, 128), synth.seed_of(77, 0, synth.T_V), DEV)
    uni = mk.MiniKVCache(B, Hkv, 1088, R=32, Hq=Hq)
    mk.quant_pack(uni, k, v)
    rag = mk.MiniKVCache(B, Hkv, 1088, R=32, Hq=Hq).set_ragged()
    for b in range(B):
        mk.quant_pack_seq(rag, b, k[b].contiguous(), v[b].contiguous())
    for s in range(steps):
        q, kn, vn = _step_inputs(B, Hq, Hkv, 78, s)
        assert torch.equal(mk.decode_attn(uni, q, kn, vn), mk.decode_attn(rag, q, kn, vn)), s
    a, c = uni.arrays(), rag.arrays()
    for name in a:
        assert torch.equal(a[name], c[name]), name
    assert all(rag.seq_state(b) == (uni.n_packed, uni.n_res, uni.res_start) for b in range(B))


def test_ragged_mass_and_static_decode():
    """decode_attn_mass and decode_attn_static step every sequence from its own state."""
    lengths, Hq, Hkv, G, R, steps = (400, 50, 1200), 4, 2, 32, 32, 12
    B, g = len(lengths), Hq // Hkv
    cache, ref = _load(lengths, Hq, Hkv, G, R, steps, 800)
    L = cache.cap + R + G
    mass = torch.zeros((B, Hkv, L), dtype=torch.float32, device=DEV)
    acc = np.zeros((B, Hkv, L))
    for s in range(steps):
        q, kn, vn = _step_inputs(B, Hq, Hkv, 81, s)
        static = s % 3 == 2
        out = mk.decode_attn_static(cache, q, kn, vn) if static else mk.decode_attn_mass(cache, q, kn, vn, mass)
        torch.cuda.synchronize()
        qn, knn, vnn = np16(q), np16(kn), np16(vn)
        got = out.float().cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                sl = ref[b][h]
                if static:
                    o = sl.step(qn[b, h * g:(h + 1) * g], knn[b, h], vnn[b, h], TAU)
                else:
                    o = sl.step_mass(qn[b, h * g:(h + 1) * g], knn[b, h], vnn[b, h], TAU, acc[b, h])
                assert float(np.max(np.abs(got[b, h * g:(h + 1) * g] - o))) <= ATOL_OUT, (s, b, h)
        err = float(np.max(np.abs(mass.double().cpu().numpy() - acc)))
        assert err <= ATOL_MASS_PER_STEP * (s + 1) + 1e-6, (s, err)
    m = mass.double().cpu().numpy()
    for b, N in enumerate(lengths):
        n = N + steps
        assert np.all(m[b, :, n:] == 0)                       # past each sequence's tokens: untouched
        mass_steps = steps - steps // 3
        np.testing.assert_allclose(m[b, :, :n].sum(-1), g * mass_steps, rtol=1e-5)
    for b in range(B):
        _compare_seq(cache, b, ref[b])


def test_evict_pack_seq_prompts_of_different_lengths():
    """Each sequence's own prompt (its T and keep) kept and packed into its row:
    the oracle's selection on the GPU's scores, and its pack of those rows."""
    Hq = Hkv = 2
    W, G, R = 32, 32, 32
    prompts = [(512, 160), (700, 700), (300, 64), (64, 32)]    # (T, keep)
    cap = (max(min(t, kp) for t, kp in prompts) // G + 2) * G
    cache = mk.MiniKVCache(len(prompts), Hkv, cap, G=G, R=R, Hq=Hq).set_ragged()
    for b, (T, keep) in enumerate(prompts):
        q = synth.normal_fp16((1, Hq, T, 128), synth.seed_of(90 + b, 0, synth.T_Q), DEV)
        k = synth.keys_fp16((1, Hkv, T, 128), synth.seed_of(90 + b, 0, synth.T_K), DEV)
        v = synth.normal_fp16((1, Hkv, T, 128), synth.seed_of(90 + b, 0, synth.T_V), DEV)
        _, scores = mk.select_prefill(q, k, v, W)
        idx = mk.evict_pack_seq(cache, b, scores[0], k[0], v[0], W, keep)
        torch.cuda.synchronize()
        sn = scores[0].cpu().numpy().astype(np.float64)
        kn, vn = np16(k[0]), np16(v[0])
        slices = []
        for h in range(Hkv):
            sel = O.select(sn[h], W, keep)
            assert np.array_equal(idx[h].cpu().numpy(), sel), (b, h)
            slices.append(O.SliceCache.from_kept(kn[h][sel], vn[h][sel], R, G, 128))
        _compare_seq(cache, b, slices)
    # loading one row leaves the others as they were
    for b in range(len(prompts)):
        assert cache.seq_state(b)[0] + cache.seq_state(b)[1] == min(prompts[b][0], prompts[b][1])


# ------------------------------------------------- device state + CUDA graphs

@pytest.mark.parametrize("with_mass", [False, True])
def test_device_state_steps_replayed_from_one_cuda_graph(with_mass):
    """With the state on the device, one captured decode step replays correctly
    for every later step: lengths grow, flushes happen, sequences differ."""
    lengths, Hq, Hkv, G, R, steps = (300, 20, 1000, 0, 161), 8, 2, 32, 32, 40
    B, g = len(lengths), Hq // Hkv
    cache, ref = _load(lengths, Hq, Hkv, G, R, steps + 1, 900, device_state=True)
    L = cache.cap + R + G
    mass = torch.zeros((B, Hkv, L), dtype=torch.float32, device=DEV)
    acc = np.zeros((B, Hkv, L))
    q_s = torch.zeros((B, Hq, 128), dtype=torch.float16, device=DEV)
    kn_s = torch.zeros((B, Hkv, 128), dtype=torch.float16, device=DEV)
    vn_s = torch.zeros_like(kn_s)
    out_s = torch.zeros_like(q_s)

    def call():
        if with_mass:
            mk.decode_attn_mass(cache, q_s, kn_s, vn_s, mass, out=out_s)
        else:
            mk.decode_attn(cache, q_s, kn_s, vn_s, out=out_s)

    graph = None
    for s in range(steps):
        q, kn, vn = _step_inputs(B, Hq, Hkv, 91, s)
        q_s.copy_(q)
        kn_s.copy_(kn)
        vn_s.copy_(vn)
        if s == 0:
            call()                       # eager first step (also sets up the library)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                call()                   # captured, not run
        else:
            graph.replay()
        torch.cuda.synchronize()
        qn, knn, vnn = np16(q), np16(kn), np16(vn)
        got = out_s.float().cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                sl = ref[b][h]
                args = (qn[b, h * g:(h + 1) * g], knn[b, h], vnn[b, h], TAU)
                o = sl.step_mass(*args, acc[b, h]) if with_mass else sl.step(*args)
                assert float(np.max(np.abs(got[b, h * g:(h + 1) * g] - o))) <= ATOL_OUT, (s, b, h)
        if with_mass:
            err = float(np.max(np.abs(mass.double().cpu().numpy() - acc)))
            assert err <= ATOL_MASS_PER_STEP * (s + 1) + 1e-6, (s, err)
    for b in range(B):
        _compare_seq(cache, b, ref[b])
    assert cache.status() == [0] * B
    del graph


def test_device_state_refuses_a_flush_past_capacity():
    """cap leaves no room for another key group: the step that would flush
    still attends correctly, then keeps the sequence's state and sets its
    status word; the other sequence, with room, flushes normally."""
    G, R, Hq, Hkv = 32, 32, 2, 2
    lengths = (64 + 62, 62)          # r = 62 each: the second step fills the ring
    cache, ref = _load(lengths, Hq, Hkv, G, R, 0, 950, device_state=True, cap=64)
    assert [cache.seq_state(b) for b in range(2)] == [(64, 62, 0), (0, 62, 0)]
    for s in range(2):
        q, kn, vn = _step_inputs(2, Hq, Hkv, 96, s)
        out = mk.decode_attn(cache, q, kn, vn)
        torch.cuda.synchronize()
        qn, knn, vnn = np16(q), np16(kn), np16(vn)
        for b in range(2):
            for h in range(Hkv):
                o = ref[b][h].step(qn[b, h:h + 1], knn[b, h], vnn[b, h], TAU)
                assert float(np.max(np.abs(out.float().cpu().numpy()[b, h:h + 1] - o))) <= ATOL_OUT, (s, b, h)
    assert cache.seq_state(0) == (64, 63, 0) and cache.status()[0] == 1     # refused, unchanged
    assert cache.seq_state(1) == (32, 32, 32) and cache.status()[1] == 0    # flushed
    _compare_seq(cache, 1, ref[1])
    a = cache.arrays()
    for h in range(Hkv):                                                    # the full sequence's packed part intact
        np.testing.assert_array_equal(a["k_codes"][0, h, :64].cpu().numpy().view(np.uint32), ref[0][h].k_codes[:64])


def test_deterministic_mode_repeats_bit_for_bit(deterministic):
    """Fixed item-to-warp assignment: two identical calls (fresh caches, same
    inputs) give bit-identical outputs, on a shape whose CTAs hold more items
    than their warps' first two each (where the default mode claims items
    dynamically).  The default mode agrees with it to half the output
    tolerance."""
    B, Hq, Hkv, N = 4, 8, 2, 4000
    k = synth.keys_fp16((B, Hkv, N, 128), synth.seed_of(79, 0, synth.T_K), DEV)
    v = synth.normal_fp16((B, Hkv, N, 128), synth.seed_of(79, 0, synth.T_V), DEV)
    q, kn, vn = _step_inputs(B, Hq, Hkv, 80, 0)

    def run():
        c = mk.MiniKVCache(B, Hkv, 4096 + 64, R=32, Hq=Hq)
        mk.quant_pack(c, k, v)
        return mk.decode_attn(c, q, kn, vn)

    a, b = run(), run()
    assert torch.equal(a, b)
    mk.set_deterministic(False)
    d = run()
    # the fp32 sums differ in their last bits; after fp16 rounding that is at most
    # about one unit in the last place of the largest outputs (here |out| < 1)
    assert float((d.float() - a.float()).abs().max()) <= 1e-3
