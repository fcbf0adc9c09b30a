"""The five workloads at full per-layer size, through the C ABI, against the oracle.

Each test runs the launch configuration the benchmark times (same B, heads,
lengths, G, R, W, keep) on two or three sampled layers, and checks:
  * select_prefill outputs on sampled (sequence, head, row) entries and window
    scores on sampled KV heads (fp64 oracle; 2e-3 / relative 1e-3);
  * top-k indices exactly against the oracle's selection run on the GPU's own
    fp32 scores, and against the fp64 oracle scores up to the 1e-4 cut rule;
  * packed codes, scales, zeros and the fp16 residual bit-exactly on sampled
    units, before and after the decode steps (flushes included);
  * decode outputs on sampled units and steps (2e-3 max-abs); the oracle keeps
    the state of the sampled units through every step.
Inputs: seeded N(0,1) fp16 with 4 x10 outlier key channels (synth.py).
"""
import math

import numpy as np
import pytest
import torch

from bit_quantized_evicted_b200 import minikv as mk
from bit_quantized_evicted_b200 import synth
from oracle import minikv_oracle as O

pytestmark = pytest.mark.gpu

ATOL = 2e-3
TAU = 1.0 / math.sqrt(128.0)
DEV = "cuda"


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mk.lib()


def _np(t):
    return t.detach().cpu().contiguous().numpy()


def _layer_qkv(wid, layer, B, Hq, Hkv, T):
    q = torch.empty((B, Hq, T, 128), dtype=torch.float16, device=DEV)
    k = torch.empty((B, Hkv, T, 128), dtype=torch.float16, device=DEV)
    v = torch.empty_like(k)
    for b in range(B):
        q[b] = synth.normal_fp16((Hq, T, 128), synth.seed_of(wid, layer, synth.T_Q, 0, b), DEV)
        k[b] = synth.keys_fp16((Hkv, T, 128), synth.seed_of(wid, layer, synth.T_K, 0, b), DEV)
        v[b] = synth.normal_fp16((Hkv, T, 128), synth.seed_of(wid, layer, synth.T_V, 0, b), DEV)
    return q, k, v


def _step_inputs(wid, layer, step, B, Hq, Hkv):
    q = synth.normal_fp16((B, Hq, 128), synth.seed_of(wid, layer, synth.T_QDEC, step), DEV)
    kn = synth.keys_fp16((B, Hkv, 128), synth.seed_of(wid, layer, synth.T_KNEW, step), DEV)
    vn = synth.normal_fp16((B, Hkv, 128), synth.seed_of(wid, layer, synth.T_VNEW, step), DEV)
    return q, kn, vn


def _check_slice(cache, b, h, sc):
    a = cache.arrays()
    nq, G = sc.n_q, cache.G
    assert cache.n_packed == nq and cache.n_res == sc.r
    assert np.array_equal(_np(a["k_codes"][b, h, :nq]).view(np.uint32), sc.k_codes)
    assert np.array_equal(_np(a["v_codes"][b, h, :nq]).view(np.uint32), sc.v_codes)
    assert np.array_equal(_np(a["k_scale"][b, h, :nq // G]).view(np.uint16), sc.k_scale)
    assert np.array_equal(_np(a["k_zero"][b, h, :nq // G]).view(np.uint16), sc.k_zero)
    assert np.array_equal(_np(a["v_scale"][b, h, :nq]).view(np.uint16), sc.v_scale)
    assert np.array_equal(_np(a["v_zero"][b, h, :nq]).view(np.uint16), sc.v_zero)
    kr, vr = cache.residual()
    assert np.array_equal(_np(kr[b, h]).view(np.uint16), np.array(sc.res_k, np.uint16).reshape(sc.r, 128))
    assert np.array_equal(_np(vr[b, h]).view(np.uint16), np.array(sc.res_v, np.uint16).reshape(sc.r, 128))


def _prefill_and_keep(wid, layer, B, Hq, Hkv, T, W, keep, G, R, sample_heads, sample_rows, sample_kv, cap_extra):
    """select_prefill -> topk_evict -> quant_pack for one layer, checked on samples.
    Returns the cache and the oracle slices of the sampled units."""
    g = Hq // Hkv
    q, k, v = _layer_qkv(wid, layer, B, Hq, Hkv, T)
    o, scores = mk.select_prefill(q, k, v, W)
    idx, kk, vk = mk.topk_evict(scores, k, v, W, keep)
    n = min(keep, T)
    cap = ((n + cap_extra) // G + 2) * G
    cache = mk.MiniKVCache(B, Hkv, cap, G=G, R=R, Hq=Hq)
    mk.quant_pack(cache, kk, vk)
    torch.cuda.synchronize()
    # prefill attention rows
    for (b, h) in sample_heads:
        ref = O.prefill_attention_rows(_np(q[b, h]), _np(k[b, h // g]), _np(v[b, h // g]), sample_rows, TAU)
        got = o[b, h, sample_rows].float().cpu().numpy()
        assert np.max(np.abs(got - ref)) <= ATOL, (layer, b, h)
    # window scores and selection
    sg = _np(scores).astype(np.float64)
    gi = _np(idx)
    for b in range(B):
        for hk in range(Hkv):
            assert np.array_equal(gi[b, hk], O.select(sg[b, hk], W, keep)), (layer, b, hk)
    for (b, hk) in sample_kv:
        sref = O.window_scores(_np(q[b, hk * g:(hk + 1) * g]), _np(k[b, hk]), W, TAU)
        assert np.all(np.abs(sg[b, hk] - sref) <= 1e-3 * np.abs(sref) + 1e-6), (layer, b, hk)
        if keep < T:
            oi = O.select(sref, W, keep)
            diff = set(oi.tolist()) ^ set(gi[b, hk].tolist())
            cut = np.sort(sref[: T - W])[::-1][keep - W - 1] if keep > W else np.inf
            assert all(abs(sref[j] - cut) < 1e-4 for j in diff), (layer, b, hk, len(diff))
        assert np.array_equal(_np(kk[b, hk]), _np(k[b, hk])[gi[b, hk]])
    slices = {(b, hk): O.SliceCache.from_kept(_np(kk[b, hk]), _np(vk[b, hk]), R, G, 128) for (b, hk) in sample_kv}
    for (b, hk), sc in slices.items():
        _check_slice(cache, b, hk, sc)
    del q, k, v, o, scores, idx, kk, vk
    return cache, slices


def _packed_cache(wid, layer, B, Hkv, N, G, R, steps):
    """An 'already packed' cache: N kept tokens per unit generated directly."""
    k = torch.empty((B, Hkv, N, 128), dtype=torch.float16, device=DEV)
    v = torch.empty_like(k)
    for b in range(B):
        k[b] = synth.keys_fp16((Hkv, N, 128), synth.seed_of(wid, layer, synth.T_K, 0, b), DEV)
        v[b] = synth.normal_fp16((Hkv, N, 128), synth.seed_of(wid, layer, synth.T_V, 0, b), DEV)
    cap = ((N + steps) // G + 2) * G
    cache = mk.MiniKVCache(B, Hkv, cap, G=G, R=R)
    mk.quant_pack(cache, k, v)
    torch.cuda.synchronize()
    return cache, k, v


def _decode_steps(wid, layer, cache, slices, B, Hq, Hkv, steps, check_steps):
    g = Hq // Hkv
    worst = 0.0
    for s in range(steps):
        q, kn, vn = _step_inputs(wid, layer, s, B, Hq, Hkv)
        out = mk.decode_attn(cache, q, kn, vn)
        check = s in check_steps
        if check:
            outn = out.float().cpu().numpy()
        qn, knn, vnn = _np(q), _np(kn), _np(vn)
        for (b, hk), sc in slices.items():
            if check:
                ref = sc.step(qn[b, hk * g:(hk + 1) * g], knn[b, hk], vnn[b, hk], TAU)
                err = float(np.max(np.abs(outn[b, hk * g:(hk + 1) * g] - ref)))
                worst = max(worst, err)
                assert err <= ATOL, (layer, s, b, hk, err)
            else:
                sc.advance(knn[b, hk], vnn[b, hk])
    torch.cuda.synchronize()
    for (b, hk), sc in slices.items():
        _check_slice(cache, b, hk, sc)
    return worst


def test_config1_tiny_layer():
    """512-token prompt, 4 MHA heads, keep 50%, W=32, G=32, R=32, one decode step."""
    B, H, T, W, keep, G, R = 1, 4, 512, 32, 256, 32, 32
    cache, slices = _prefill_and_keep(101, 0, B, H, H, T, W, keep, G, R, [(0, h) for h in range(H)],
                                      np.arange(T), [(0, h) for h in range(H)], 4)
    _decode_steps(101, 0, cache, slices, B, H, H, 1, {0})


def test_config2_llama2_7b_prefill_and_decode():
    """32 MHA heads, prompt 4096, keep 15% (614), W=32, G=32, R=128, 128 decode steps; layers 0 and 31."""
    B, H, T, W, keep, G, R, steps = 1, 32, 4096, 32, 4096 * 15 // 100, 32, 128, 128
    rows = np.array([0, 1, 2, 63, 64, 65, 1000, 2047, 4031, 4064, 4095])
    for layer in (0, 31):
        cache, slices = _prefill_and_keep(102, layer, B, H, H, T, W, keep, G, R, [(0, 0), (0, 17), (0, 31)],
                                          rows, [(0, h) for h in range(H)], steps)
        assert (cache.n_packed, cache.n_res) == (480, 134)
        _decode_steps(102, layer, cache, slices, B, H, H, steps, set(range(steps)))


@pytest.mark.parametrize("wid,B,Hq,Hkv,N,steps", [
    (103, 8, 40, 40, 16384 * 15 // 100, 256),   # LLaMA2-13B-shaped MHA decode
    (104, 16, 32, 8, 32768 * 20 // 100, 256),   # Mistral-7B-shaped GQA decode
])
def test_config3_4_packed_decode(wid, B, Hq, Hkv, N, steps):
    G, R = 32, 128
    units = [(0, 0), (B // 2, Hkv // 2), (B - 1, Hkv - 1)]
    checks = {0, 5, 6, 7, 38, 100, steps - 1}
    for layer in (0, 1):
        cache, k, v = _packed_cache(wid, layer, B, Hkv, N, G, R, steps)
        assert (cache.n_packed, cache.n_res) == ((2304, 153) if wid == 103 else (6400, 153))
        slices = {(b, h): O.SliceCache.from_kept(_np(k[b, h]), _np(v[b, h]), R, G, 128) for (b, h) in units}
        for (b, h), sc in slices.items():
            _check_slice(cache, b, h, sc)
        del k, v
        _decode_steps(wid, layer, cache, slices, B, Hq, Hkv, steps, checks)


def test_quant_only_32k_decode():
    """The keep-100 % (quantization only) workload at its own size: Mistral-7B GQA
    shape, all 32768 context tokens kept (32640 packed + 128 fp16 per unit), 40
    decode steps crossing a key-group flush at step 31, two layers, sampled
    units.  It has the most packed tokens per unit of any workload, so the most
    CTAs meet in each unit's split-KV merge."""
    wid, B, Hq, Hkv, N, steps = 106, 16, 32, 8, 32768, 40
    G, R = 32, 128
    units = [(0, 0), (7, 3), (B - 1, Hkv - 1)]
    for layer in (0, 1):
        cache, k, v = _packed_cache(wid, layer, B, Hkv, N, G, R, steps)
        assert (cache.n_packed, cache.n_res) == (32640, 128)
        slices = {(b, h): O.SliceCache.from_kept(_np(k[b, h]), _np(v[b, h]), R, G, 128) for (b, h) in units}
        for (b, h), sc in slices.items():
            _check_slice(cache, b, h, sc)
        del k, v
        _decode_steps(wid, layer, cache, slices, B, Hq, Hkv, steps, {0, 1, 30, 31, 32, steps - 1})
        assert cache.n_packed == 32640 + G   # one key group was flushed in every unit
        del cache
        torch.cuda.empty_cache()


def test_pyramid_max_batch_decode():
    """The long-prompt pyramid workload at the largest batch that fits the free
    HBM (the bench's own sizing rule), in the launch configuration the bench
    times (per-sequence state on the GPU): layer 0 (keep 13200 of 44000), every
    sequence loaded, 3 decode steps, sampled units against the oracle."""
    import bench
    wid, H, T, G, R, steps = 107, 32, 44000, 32, 128, 3
    free, _ = torch.cuda.mem_get_info()
    B, _ = bench.max_batch(mk, free, preset=bench.DECODE_PRESETS["pyramid_44k_maxbatch_decode"])
    assert B >= 64   # ~0.75 GB per sequence for all 32 layers: well over 64 fit in 180 GB
    N = O.pyramid_keep(T, 0, 32)
    cap = ((N + 512 + 8) // G + 2) * G
    cache = mk.MiniKVCache(B, H, cap, G=G, R=R, Hq=H).set_device_state()
    units = [(0, 0), (B // 2, 17), (B - 1, H - 1)]
    slices = {}
    for b in range(B):
        kb = synth.keys_fp16((H, N, 128), synth.seed_of(wid, 0, synth.T_K, 0, b), DEV)
        vb = synth.normal_fp16((H, N, 128), synth.seed_of(wid, 0, synth.T_V, 0, b), DEV)
        mk.quant_pack_seq(cache, b, kb, vb)
        for (ub, h) in units:
            if ub == b:
                slices[(b, h)] = O.SliceCache.from_kept(_np(kb[h]), _np(vb[h]), R, G, 128)
        del kb, vb
    for s in range(steps):
        q, kn, vn = _step_inputs(wid, 0, s, B, H, H)
        out = mk.decode_attn(cache, q, kn, vn)
        outn, qn, knn, vnn = out.float().cpu().numpy(), _np(q), _np(kn), _np(vn)
        for (b, h), sc in slices.items():
            ref = sc.step(qn[b, h:h + 1], knn[b, h], vnn[b, h], TAU)
            err = float(np.max(np.abs(outn[b, h:h + 1] - ref)))
            assert err <= ATOL, (s, b, h, err)
    torch.cuda.synchronize()
    assert cache.status() == [0] * B
    for (b, h), sc in slices.items():
        assert cache.seq_state(b)[:2] == (sc.n_q, sc.r)
    del cache
    torch.cuda.empty_cache()


def test_config5_pyramid_long_prompt():
    """LLaMA2-7B shape, B=4, prompt 44000, keep from 30% (layer 0) to 5% (layer 31), W=32, G=32, R=128,
    prefill select + pack + 512 decode steps on layers 0, 15 and 31."""
    B, H, T, W, G, R, steps = 4, 32, 44000, 32, 32, 128, 512
    rows = np.array([0, 1, 31, 32, 5000, 43967, 43968, 43999])
    for layer in (0, 15, 31):
        keep = O.pyramid_keep(T, layer, 32)
        cache, slices = _prefill_and_keep(105, layer, B, H, H, T, W, keep, G, R, [(0, 0), (3, 31)], rows,
                                          [(0, 0), (2, 13), (3, 31)], steps)
        _decode_steps(105, layer, cache, slices, B, H, H, steps, {0, 7, 200, steps - 1})
        del cache
        torch.cuda.empty_cache()
