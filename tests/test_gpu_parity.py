"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: packed codes, scales, zeros, the fp16 residual and kept indices are
bit-exact; attention outputs (fp16) are within 2e-3 max-abs of the oracle's
fp64 result; window scores (fp32) within a relative 1e-3 (+1e-6); running
attention masses within 2e-5 per accumulated step.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from bit_quantized_evicted_b200 import minikv as mk
from bit_quantized_evicted_b200 import synth
from oracle import minikv_oracle as O
from tests.oracle_runs import (compare_cache, decode_mass_reference_step, decode_reference_step, np16,
                               pack_reference, prefill_reference)

pytestmark = pytest.mark.gpu

ATOL_OUT = 2e-3
TAU = 1.0 / math.sqrt(128.0)
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mk.lib()


def _kv(B, H, N, seed, device=DEV):
    k = synth.keys_fp16((B, H, N, 128), synth.seed_of(seed, 0, synth.T_K), device)
    v = synth.normal_fp16((B, H, N, 128), synth.seed_of(seed, 0, synth.T_V), device)
    return k, v


# ------------------------------------------------------------------ pack

@pytest.mark.parametrize("B,H,N,G,Gv,R,cap", [
    (1, 4, 256, 32, 128, 32, 256),     # 512-token prompt, keep 50%
    (2, 3, 300, 32, 64, 48, 320),      # ragged: residual 60, Gv = 64
    (1, 2, 20, 32, 128, 32, 64),       # shorter than R: all residual
    (1, 1, 160 + 128 + 50, 64, 16, 128, 256),
    (1, 2, 0, 32, 128, 32, 64),        # empty
    (3, 2, 32 * 40 + 31, 32, 128, 0, 32 * 40 + 32),   # R = 0
    (1, 2, 32 * 8 + 40, 32, 32, 32, 320),             # Gv = 32
    (1, 1, 128 * 3 + 100, 128, 128, 64, 512),         # G = 128: one block per group
    (4, 8, 32 * 40 + 40, 32, 128, 32, 32 * 41),       # 1280 groups: blocks pack several, double-buffered
    (2, 8, 64 * 60 + 100, 64, 64, 64, 64 * 61),       # the same at G = 64
])
def test_quant_pack_bitexact(B, H, N, G, Gv, R, cap):
    k, v = _kv(B, H, N, 101 + N)
    if N >= 64:   # degenerate groups: constant, zeros with -0, huge range
        k[0, 0, :32, 5] = 0.75
        k[0, 0, :32, 6] = 0.0
        k[0, 0, 3, 6] = -0.0
        v[0, 0, 1, :] = -2.5
        k[0, 0, 32:64, 7] = torch.linspace(-60000, 60000, 32, dtype=torch.float32).half()
    cache = mk.MiniKVCache(B, H, cap, G=G, Gv=Gv, R=R)
    mk.quant_pack(cache, k, v)
    torch.cuda.synchronize()
    ref = pack_reference(k, v, R, G, Gv)
    compare_cache(cache, ref)


# ------------------------------------------------------- select prefill

@pytest.mark.parametrize("B,Hq,Hkv,T,W,kind", [(c + ("plain",))[:6] for c in [
    (1, 4, 4, 512, 32),      # tiny single layer
    (1, 8, 2, 300, 17),      # GQA, ragged tail
    (2, 2, 1, 130, 130),     # window = whole prompt
    (1, 1, 1, 1, 1),
    (1, 4, 1, 200, 32),      # g = 4
    (1, 2, 1, 1000, 32),     # 8 query tiles, key-block stages reused
    (2, 4, 2, 2100, 64),     # 17 tiles, ragged last tile
    (1, 2, 2, 1500, 32, "ramp"),   # key norms growing with position: the running max moves late
]])
def test_select_prefill_vs_oracle(B, Hq, Hkv, T, W, kind):
    q = synth.normal_fp16((B, Hq, T, 128), synth.seed_of(7, T, synth.T_Q), DEV)
    k, v = _kv(B, Hkv, T, 7 + T)
    if kind == "ramp":
        ramp = 1.0 + 4.0 * torch.arange(T, device=DEV, dtype=torch.float32) / T
        k = (k.float() * ramp[None, None, :, None]).half()
    o, scores = mk.select_prefill(q, k, v, W)
    torch.cuda.synchronize()
    outs, sref = prefill_reference(q, k, v, W, TAU)
    on = o.float().cpu().numpy()
    err = max(np.max(np.abs(on[b, h] - ref)) for (b, h), ref in outs.items())
    assert err <= ATOL_OUT, err
    sg = scores.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(sg - sref) <= 1e-3 * np.abs(sref) + 1e-6), np.max(np.abs(sg - sref))
    g = Hq // Hkv
    np.testing.assert_allclose(sg.sum(-1), W * g, rtol=1e-4)


# ------------------------------------------------------- fused evict + pack

@pytest.mark.parametrize("B,H,T,W,keep,G,R", [
    (1, 4, 512, 32, 256, 32, 32),     # tiny layer, keep 50%
    (2, 3, 1000, 16, 150, 32, 48),    # ragged residual
    (1, 2, 300, 32, 300, 64, 128),    # keep = T: every row, G = 64
    (1, 2, 64, 32, 32, 32, 32),       # only the window, all residual
])
def test_evict_pack_matches_topk_then_pack(B, H, T, W, keep, G, R):
    """evict_pack == quant_pack(topk_evict(...)) bit for bit, and both == the oracle's pack of its selection."""
    scores = torch.rand((B, H, T), generator=torch.Generator().manual_seed(T + keep), dtype=torch.float32).to(DEV)
    k, v = _kv(B, H, T, 500 + T)
    n = min(keep, T)
    cap = (n // G + 2) * G
    idx, kk, vk = mk.topk_evict(scores, k, v, W, keep)
    ref_cache = mk.MiniKVCache(B, H, cap, G=G, R=R)
    mk.quant_pack(ref_cache, kk, vk)
    cache = mk.MiniKVCache(B, H, cap, G=G, R=R)
    idx2 = mk.evict_pack(cache, scores, k, v, W, keep)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert (cache.n_packed, cache.n_res, cache.res_start) == (ref_cache.n_packed, ref_cache.n_res, 0)
    a, b = cache.arrays(), ref_cache.arrays()
    nq = cache.n_packed
    for name in ("k_codes", "v_codes", "v_scale", "v_zero"):
        assert torch.equal(a[name][:, :, :nq], b[name][:, :, :nq]), name
    for name in ("k_scale", "k_zero"):
        assert torch.equal(a[name][:, :, :nq // G], b[name][:, :, :nq // G]), name
    kr, vr = cache.residual()
    kr2, vr2 = ref_cache.residual()
    assert torch.equal(kr, kr2) and torch.equal(vr, vr2)
    # and against the oracle: its selection on the same scores, its pack of those rows
    sn = scores.cpu().numpy().astype(np.float64)
    for b_ in range(B):
        for h in range(H):
            sel = O.select(sn[b_, h], W, keep)
            assert np.array_equal(idx2[b_, h].cpu().numpy(), sel)
    ref = pack_reference(kk, vk, R, G, 128)
    compare_cache(cache, ref)


# ------------------------------------------------------------- top-k

def _select_ref(scores_np, W, keep):
    B, H, T = scores_np.shape
    return np.stack([np.stack([O.select(scores_np[b, h], W, keep) for h in range(H)]) for b in range(B)])


@pytest.mark.parametrize("B,H,T,W,keep", [
    (1, 4, 512, 32, 256),
    (2, 3, 1000, 16, 150),
    (1, 2, 300, 0, 45),
    (1, 2, 64, 32, 32),       # keep = W: only the window
    (1, 2, 64, 8, 64),        # keep = T
    (1, 1, 50, 8, 500),       # keep > T
    (1, 2, 44000, 32, 13200),
])
def test_topk_exact_with_ties(B, H, T, W, keep):
    gen = torch.Generator().manual_seed(T + keep)
    s = (torch.randint(0, 9, (B, H, T), generator=gen).float() / 7.0)   # many exact ties
    s[..., ::17] = torch.rand((B, H, (T + 16) // 17), generator=gen)
    s = s.to(DEV)
    k, v = _kv(B, H, T, 55)
    idx, kk, vk = mk.topk_evict(s, k, v, W, keep)
    torch.cuda.synchronize()
    ref = _select_ref(s.cpu().numpy(), W, keep)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    ri = torch.from_numpy(ref).long().to(DEV)
    assert torch.equal(kk, torch.gather(k, 2, ri[..., None].expand(-1, -1, -1, 128)))
    assert torch.equal(vk, torch.gather(v, 2, ri[..., None].expand(-1, -1, -1, 128)))


@pytest.mark.parametrize("T,W,keep", [(2, 0, 1), (300, 8, 40), (1000, 16, 700), (4100, 32, 600)])
def test_topk_signed_zeros_tie(T, W, keep):
    """-0 and +0 are the same score: among them the lower index is kept,
    exactly as the oracle (which compares the scores as numbers) keeps it."""
    gen = torch.Generator().manual_seed(T)
    s = torch.randint(0, 3, (1, 2, T), generator=gen).float() / 4.0   # many exact ties
    zeros = torch.rand((1, 2, T), generator=gen) < 0.5
    sign = torch.where(torch.rand((1, 2, T), generator=gen) < 0.5, -1.0, 1.0)
    s = torch.where(zeros, sign * 0.0, s)   # about half the scores are -0 or +0
    if T == 2:
        s[0, :, 0], s[0, :, 1] = -0.0, 0.0   # [-0, +0], keep 1: index 0
    s = s.to(DEV)
    k, v = _kv(1, 2, T, 57)
    idx, kk, vk = mk.topk_evict(s, k, v, W, keep)
    torch.cuda.synchronize()
    ref = _select_ref(s.cpu().numpy(), W, keep)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    if T == 2:
        assert idx.cpu().numpy()[0, :, 0].tolist() == [0, 0]


# ------------------------------------------------------------- decode

@pytest.mark.parametrize("B,Hq,Hkv,N,G,R,steps", [
    (1, 4, 4, 256, 32, 32, 36),      # tiny single layer; crosses a flush
    (2, 8, 2, 1000, 32, 128, 8),     # GQA g = 4
    (1, 2, 2, 4000, 32, 128, 3),     # many packed chunks per KV head
    (1, 3, 1, 20, 32, 32, 3),        # nothing packed yet; g = 3
    (2, 4, 2, 700, 64, 64, 70),      # G = 64, two flushes
    (1, 2, 2, 96, 32, 0, 40),        # R = 0: every 32 steps the whole residual is packed
])
def test_decode_vs_oracle(B, Hq, Hkv, N, G, R, steps):
    Gv = 128
    k, v = _kv(B, Hkv, N, 300 + N)
    cap = ((N + steps) // G + 2) * G
    cache = mk.MiniKVCache(B, Hkv, cap, G=G, Gv=Gv, R=R, Hq=Hq)
    mk.quant_pack(cache, k, v)
    ref = pack_reference(k, v, R, G, Gv)
    worst = 0.0
    for s in range(steps):
        q = synth.normal_fp16((B, Hq, 128), synth.seed_of(9, N, synth.T_QDEC, s), DEV)
        kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(9, N, synth.T_KNEW, s), DEV)
        vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(9, N, synth.T_VNEW, s), DEV)
        out = mk.decode_attn(cache, q, kn, vn)
        torch.cuda.synchronize()
        oref = decode_reference_step(ref, q, kn, vn, TAU)
        err = float(np.max(np.abs(out.float().cpu().numpy() - oref)))
        worst = max(worst, err)
        assert err <= ATOL_OUT, (s, err)
    compare_cache(cache, ref)       # flushes packed bit-exactly
    print(f"decode max-abs error {worst:.2e}")


# Attention mass: each step adds g probabilities per KV head; the kernel's
# log2 scores carry fp32 accumulation and ex2.approx error (relative ~1e-6 on
# each probability), so the running sums may drift by a few 1e-6 per step.
ATOL_MASS_PER_STEP = 2e-5


@pytest.mark.parametrize("B,Hq,Hkv,N,G,R,steps", [
    (1, 4, 4, 256, 32, 32, 36),      # g = 1; crosses a flush
    (2, 8, 2, 1000, 32, 128, 8),     # GQA g = 4, several packed CTAs per KV head
    (1, 3, 1, 20, 32, 32, 3),        # nothing packed yet; g = 3
    (1, 2, 2, 96, 32, 0, 40),        # R = 0: the whole residual is packed every 32 steps
    (2, 4, 2, 700, 64, 64, 70),      # G = 64, two flushes, g = 2
])
def test_decode_mass_vs_oracle(B, Hq, Hkv, N, G, R, steps):
    Gv = 128
    g = Hq // Hkv
    k, v = _kv(B, Hkv, N, 500 + N)
    cap = ((N + steps) // G + 2) * G
    cache = mk.MiniKVCache(B, Hkv, cap, G=G, Gv=Gv, R=R, Hq=Hq)
    mk.quant_pack(cache, k, v)
    ref = pack_reference(k, v, R, G, Gv)
    L = cap + R + G
    # running scores start non-zero: the call adds, it does not overwrite
    mass0 = torch.rand((B, Hkv, L), generator=torch.Generator().manual_seed(N), dtype=torch.float64)
    acc = mass0.numpy().copy()
    mass = mass0.float().to(DEV)
    for s in range(steps):
        q = synth.normal_fp16((B, Hq, 128), synth.seed_of(11, N, synth.T_QDEC, s), DEV)
        kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(11, N, synth.T_KNEW, s), DEV)
        vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(11, N, synth.T_VNEW, s), DEV)
        out = mk.decode_attn_mass(cache, q, kn, vn, mass)
        torch.cuda.synchronize()
        oref = decode_mass_reference_step(ref, q, kn, vn, TAU, acc)
        assert float(np.max(np.abs(out.float().cpu().numpy() - oref))) <= ATOL_OUT, s
        got = mass.double().cpu().numpy()
        err = float(np.max(np.abs(got - acc)))
        assert err <= ATOL_MASS_PER_STEP * (s + 1) + 1e-6, (s, err)
    n = N + steps
    got = mass.double().cpu().numpy()
    np.testing.assert_array_equal(got[:, :, n:], mass0.float().double().numpy()[:, :, n:])   # untouched
    np.testing.assert_allclose((got - mass0.float().double().numpy())[:, :, :n].sum(-1), g * steps, rtol=1e-5)
    compare_cache(cache, ref)


def test_decode_mass_argument_errors():
    """Bad arguments are refused before anything is queued: the cache state and
    the running scores stay as they were."""
    B, Hq, Hkv = 1, 4, 2
    cache = mk.MiniKVCache(B, Hkv, 128, R=32, Hq=Hq)
    k, v = _kv(B, Hkv, 100, 7)
    mk.quant_pack(cache, k, v)
    q = torch.zeros((B, Hq, 128), dtype=torch.float16, device=DEV)
    kn = torch.zeros((B, Hkv, 128), dtype=torch.float16, device=DEV)
    out = torch.empty_like(q)
    mass = torch.zeros((B, Hkv, 128 + 32 + 32), dtype=torch.float32, device=DEV)
    small = torch.zeros(64, dtype=torch.uint8, device=DEV)
    with pytest.raises(mk.MiniKVError) as e:
        mk.decode_attn_mass(cache, q, kn, kn, mass, ws=small)
    assert e.value.code == mk.ERR_INVALID_ARG
    ws = torch.zeros(mk.workspace_size(mk.OP_DECODE_ATTN_MASS, B, Hq, Hkv, 192), dtype=torch.uint8, device=DEV)
    L = mk.lib()
    s = torch.cuda.current_stream().cuda_stream
    for bad_mass in (None, mass.data_ptr() + 2):
        rc = L.minikv_decode_attn_mass(ctypes.byref(cache.c), q.data_ptr(), kn.data_ptr(), kn.data_ptr(), Hq,
                                       TAU, out.data_ptr(), bad_mass, ws.data_ptr(), ws.numel(), s)
        assert rc == mk.ERR_INVALID_ARG
    assert (cache.n_packed, cache.n_res) == (64, 36)
    torch.cuda.synchronize()
    assert float(mass.abs().sum()) == 0.0


def test_decode_workspace_reuse_across_layers():
    """Two caches sharing one workspace, calls interleaved on one stream: the
    arrival counters reset themselves, so results stay exact."""
    B, Hq, Hkv, N = 2, 8, 2, 500
    ws = torch.zeros(mk.workspace_size(mk.OP_DECODE_ATTN, B, Hq, Hkv, 1024), dtype=torch.uint8, device=DEV)
    caches, refs = [], []
    for layer in range(2):
        k, v = _kv(B, Hkv, N, 900 + layer)
        c = mk.MiniKVCache(B, Hkv, 640, R=128, Hq=Hq, ws=ws)
        mk.quant_pack(c, k, v)
        caches.append(c)
        refs.append(pack_reference(k, v, 128, 32, 128))
    for s in range(3):
        for layer in range(2):
            q = synth.normal_fp16((B, Hq, 128), synth.seed_of(10, layer, synth.T_QDEC, s), DEV)
            kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(10, layer, synth.T_KNEW, s), DEV)
            vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(10, layer, synth.T_VNEW, s), DEV)
            out = mk.decode_attn(caches[layer], q, kn, vn)
            oref = decode_reference_step(refs[layer], q, kn, vn, TAU)
            assert float(np.max(np.abs(out.float().cpu().numpy() - oref))) <= ATOL_OUT
    assert int(ws[:4 * B * Hkv].view(torch.int32).abs().sum()) == 0


# ---------------------------------------------------------- whole path

def test_pipeline_tiny_layer_end_to_end():
    """512-token prompt, 4 heads: select_prefill -> topk_evict (keep 50%, W=32)
    -> quant_pack (G=32, R=32) -> one decode step, each against the oracle."""
    B, H, T, W, keep, G, Gv, R = 1, 4, 512, 32, 256, 32, 128, 32
    q = synth.normal_fp16((B, H, T, 128), synth.seed_of(1, 0, synth.T_Q), DEV)
    k = synth.keys_fp16((B, H, T, 128), synth.seed_of(1, 0, synth.T_K), DEV)
    v = synth.normal_fp16((B, H, T, 128), synth.seed_of(1, 0, synth.T_V), DEV)
    o, scores = mk.select_prefill(q, k, v, W)
    idx, kk, vk = mk.topk_evict(scores, k, v, W, keep)
    cache = mk.MiniKVCache(B, H, 512, G=G, Gv=Gv, R=R)
    mk.quant_pack(cache, kk, vk)
    qd = synth.normal_fp16((B, H, 128), synth.seed_of(1, 0, synth.T_QDEC), DEV)
    kn = synth.keys_fp16((B, H, 128), synth.seed_of(1, 0, synth.T_KNEW), DEV)
    vn = synth.normal_fp16((B, H, 128), synth.seed_of(1, 0, synth.T_VNEW), DEV)
    out = mk.decode_attn(cache, qd, kn, vn)
    torch.cuda.synchronize()

    outs, sref = prefill_reference(q, k, v, W, TAU)
    assert max(np.max(np.abs(o.float().cpu().numpy()[b, h] - r)) for (b, h), r in outs.items()) <= ATOL_OUT
    # kept sets: identical except where the oracle's scores sit within 1e-4 of the cut
    gi = idx.cpu().numpy()
    for h in range(H):
        oi = O.select(sref[0, h], W, keep)
        diff = set(oi) ^ set(gi[0, h])
        cand = np.sort(sref[0, h, : T - W])[::-1]
        cut = cand[keep - W - 1]
        assert all(abs(sref[0, h, j] - cut) < 1e-4 for j in diff), (h, diff)
    # downstream stages take the GPU's kept set as their input
    ref = pack_reference(kk, vk, R, G, Gv)
    oref = decode_reference_step(ref, qd, kn, vn, TAU)
    compare_cache(cache, ref)
    assert float(np.max(np.abs(out.float().cpu().numpy() - oref))) <= ATOL_OUT
