"""Pins for the CPU oracle (no GPU).

Each test ties one oracle step to something other than the oracle itself:
numpy's fp16 rounding, torch's fp64 attention, a closed form, an invariant or
brute force on a tiny input.  The steps are those of the MiniKV method as the
pages name them (abstract; gptget.net summary, 方法论 / 方法详解), restated in
oracle/minikv_oracle.c as O1..O10.
"""
import math

import numpy as np
import pytest
import torch

from bit_quantized_evicted_b200 import synth

TAU = 1.0 / math.sqrt(128.0)


def f16(a):
    return np.asarray(a, dtype=np.float16)


# ------------------------------------------------------------------ fp16

def test_half_to_double_exhaustive(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = oracle.half_to_double(bits)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite], ref[finite])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_float_to_half_matches_numpy(oracle):
    rng = np.random.default_rng(1)
    # every float32 exponent that can reach fp16, random mantissas
    mant = rng.integers(0, 1 << 23, 60000, dtype=np.uint32)
    expo = rng.integers(100, 145, 60000, dtype=np.uint32)
    sign = rng.integers(0, 2, 60000, dtype=np.uint32)
    x = ((sign << 31) | (expo << 23) | mant).astype(np.uint32).view(np.float32)
    # exact ties between neighbouring fp16 values, subnormal edges, overflow edge
    h = rng.integers(0, 0x7bff, 4000).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float32)
    hi = (h + 1).view(np.float16).astype(np.float32)
    ties = ((lo.astype(np.float64) + hi.astype(np.float64)) / 2).astype(np.float32)
    edges = np.array([0.0, -0.0, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.5, 2.0 ** -26, 2.0 ** -14,
                      2.0 ** -14 - 2.0 ** -25, 65504.0, 65519.99, 65520.0, 1e6, -65520.0],
                     dtype=np.float32)
    allx = np.concatenate([x, ties, edges])
    with np.errstate(over="ignore"):
        ref = allx.astype(np.float16).view(np.uint16)
    got = oracle.float_to_half(allx)
    assert np.array_equal(got, ref)


# ------------------------------------------------------- O6 quantizer

def _groups(rng):
    out = []
    for n in (32, 128):
        for _ in range(150):
            out.append(f16(rng.standard_normal(n)))
        for _ in range(40):
            out.append(f16(rng.standard_normal(n) * 10))
        for _ in range(20):
            out.append(f16(rng.standard_normal(n) * 1e-6))           # fp16 subnormals
        for _ in range(10):
            out.append(f16(rng.uniform(-60000, 60000, n)))
        for _ in range(10):
            out.append(f16(rng.choice([-1.5, 2.25], n)))              # two values
        out.append(f16(np.full(n, 0.75)))
        out.append(f16(np.concatenate([np.full(n - 1, -0.0), [0.0]])))
    return out


def test_quantizer_invariants_and_nearest_level(oracle):
    """codes in [0,3]; zero = min; scale = fp16(fp32(max-min)/3) by numpy's own
    rounding; min -> code 0 and max -> code 3; the code is the nearest of the
    four levels (fp64 brute force) except within 1e-6*scale of a midpoint;
    |x - x^| <= scale/2*(1+2^-9) + 2^-24."""
    rng = np.random.default_rng(2)
    for x in _groups(rng):
        s_bits, z_bits, codes = oracle.quantize_group(x)
        xd = x.astype(np.float64)
        s = np.uint16(s_bits).view(np.float16).astype(np.float64)
        z = np.uint16(z_bits).view(np.float16).astype(np.float64)
        assert codes.min() >= 0 and codes.max() <= 3
        assert z == xd.min()
        mx32, mn32 = np.float32(x.max()) + 0, np.float32(x.min()) + 0   # -0 -> +0
        assert s_bits == np.float16(np.float32(mx32 - mn32) / np.float32(3)).view(np.uint16)
        xhat = codes * s + z
        assert np.all(np.abs(xd - xhat) <= s / 2 * (1 + 2.0 ** -9) + 2.0 ** -24)
        if s == 0:
            assert np.all(codes == 0)
            continue
        assert codes[np.argmin(xd)] == 0 and codes[np.argmax(xd)] == 3
        levels = np.arange(4)[None, :] * s + z
        dist = np.abs(xd[:, None] - levels)
        best = np.argmin(dist, axis=1)
        srt = np.sort(dist, axis=1)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-6 * s
        assert np.array_equal(codes[clear], best[clear])


def test_quantizer_constant_group(oracle):
    for v in (0.0, 1.0, -3.5, 60000.0, 2.0 ** -24):
        x = f16(np.full(32, v))
        s_bits, z_bits, codes = oracle.quantize_group(x)
        assert s_bits == 0 and np.all(codes == 0)
        assert np.uint16(z_bits).view(np.float16) == np.float16(v)


def test_quantizer_negative_zero_minimum_stored_as_plus_zero(oracle):
    x = f16([-0.0, 0.5, 1.0, 0.25])
    _, z_bits, _ = oracle.quantize_group(x)
    assert z_bits == 0x0000


def test_quantizer_exact_ramp(oracle):
    """x = zero + c*s with fp16-exact s and zero: codes are c and x^ == x exactly."""
    rng = np.random.default_rng(3)
    for s in (0.25, 1.0, 3.0, 0.0625, 96.0):
        for zero in (-2.0, 0.0, 5.5):
            c = rng.integers(0, 4, 32)
            c[0], c[1] = 0, 3
            x = f16(zero + c * s)
            assert np.array_equal(x.astype(np.float64), zero + c * s)
            s_bits, z_bits, codes = oracle.quantize_group(x)
            assert np.uint16(s_bits).view(np.float16) == np.float16(s)
            assert np.array_equal(codes, c)


def test_quantizer_exact_half_way_quotients_round_to_even(oracle):
    """Groups whose (x - zero)/scale lands exactly on 0.5, 1.5 and 2.5: the
    reading of the quantizer rounds those ties to even, so the codes are
    0, 2, 2 (rounding half away from zero would give 1, 2, 3).  Every value,
    the scale and (x - zero)/scale are exact in fp16/fp32, so the expected
    codes below are written by hand."""
    cases = [
        # zero, scale, x / scale offsets from zero, expected codes
        (0.0, 0.25, [0.0, 0.5, 1.5, 2.5, 3.0, 1.0, 2.0], [0, 0, 2, 2, 3, 1, 2]),
        (-1.0, 0.5, [0.0, 0.5, 1.5, 2.5, 3.0], [0, 0, 2, 2, 3]),
        (2.0, 3.0, [0.0, 0.5, 1.5, 2.5, 3.0], [0, 0, 2, 2, 3]),
        (-6.0, 0.0625, [3.0, 2.5, 0.5, 1.5, 0.0, 2.5], [3, 2, 0, 2, 0, 2]),
    ]
    for zero, s, offs, want in cases:
        xd = zero + np.asarray(offs) * s
        x = f16(xd)
        assert np.array_equal(x.astype(np.float64), xd)   # exact in fp16
        s_bits, z_bits, codes = oracle.quantize_group(x)
        assert np.uint16(s_bits).view(np.float16) == np.float16(s)
        assert np.uint16(z_bits).view(np.float16) == np.float16(zero)
        assert codes.tolist() == want, (zero, s, codes.tolist())


# ------------------------------------------------------------ O7 packing

def _unpack(words, D):
    w = np.asarray(words, np.uint32)
    shifts = (2 * np.arange(16)).astype(np.uint32)
    return ((w[..., :, None] >> shifts) & 3).reshape(*w.shape[:-1], D).astype(np.uint8)


def test_pack_layout(oracle):
    codes = np.zeros(128, np.uint8)
    codes[0] = 1
    codes[17] = 3
    codes[127] = 2
    w = oracle.pack_token(codes)
    assert w[0] == 1 and w[1] == 0b1100 and w[7] == (2 << 30)
    rng = np.random.default_rng(4)
    for _ in range(50):
        c = rng.integers(0, 4, 128).astype(np.uint8)
        assert np.array_equal(_unpack(oracle.pack_token(c), 128), c)


def test_pack_tokens_groups(oracle):
    """Key groups run over G consecutive tokens per channel; value groups over Gv
    consecutive channels per token: checked against quantize_group slice by slice."""
    rng = np.random.default_rng(5)
    G, Gv, D, n = 32, 64, 128, 96
    k = synth.keys_fp16((n, D), 11).numpy()
    v = f16(rng.standard_normal((n, D)))
    p = oracle.pack_tokens(k, v, G, Gv)
    kc, vc = _unpack(p["k_codes"], D), _unpack(p["v_codes"], D)
    for g in range(n // G):
        for c in (0, 3, 4, 77, 127):
            s, z, codes = oracle.quantize_group(k[g * G:(g + 1) * G, c])
            assert p["k_scale"][g, c] == s and p["k_zero"][g, c] == z
            assert np.array_equal(kc[g * G:(g + 1) * G, c], codes)
    for t in (0, 1, 50, 95):
        for j in range(D // Gv):
            s, z, codes = oracle.quantize_group(v[t, j * Gv:(j + 1) * Gv])
            assert p["v_scale"][t, j] == s and p["v_zero"][t, j] == z
            assert np.array_equal(vc[t, j * Gv:(j + 1) * Gv], codes)


# ------------------------------------------------------------ O5 split

def test_split_closed_form(oracle):
    # keep = floor(p*T) kept tokens, residual R, key group G: the four fixed-size
    # workloads (512@50%/R32, 4096@15%, 16384@15%, 32768@20%, R128, G32)
    assert oracle.split(512 * 50 // 100, 32, 32) == (224, 32)
    assert oracle.split(4096 * 15 // 100, 128, 32) == (480, 134)
    assert oracle.split(16384 * 15 // 100, 128, 32) == (2304, 153)
    assert oracle.split(32768 * 20 // 100, 128, 32) == (6400, 153)
    for N in range(0, 400):
        nq, r = oracle.split(N, 128, 32)
        assert nq + r == N and nq % 32 == 0
        assert (r == N) if N < 128 else (128 <= r < 160)


def test_pyramid_schedule_closed_form(oracle):
    ks = [oracle.pyramid_keep(44000, l, 32) for l in range(32)]
    assert ks[0] == 13200 and ks[-1] == 2200 and sum(ks) == 246385
    assert all(a >= b for a, b in zip(ks, ks[1:]))


# ---------------------------------------------------- O1 prefill attention

def _sdpa64(q, k, v, causal):
    qt = torch.from_numpy(q.astype(np.float64))[None, None]
    kt = torch.from_numpy(k.astype(np.float64))[None, None]
    vt = torch.from_numpy(v.astype(np.float64))[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=TAU)
    return o[0, 0].numpy()


def test_prefill_attention_matches_torch_fp64(oracle):
    T, D = 77, 128
    q = synth.normal_fp16((T, D), 21).numpy()
    k = synth.keys_fp16((T, D), 22).numpy()
    v = synth.normal_fp16((T, D), 23).numpy()
    o = oracle.prefill_attention(q, k, v, TAU)
    assert np.max(np.abs(o - _sdpa64(q, k, v, True))) < 1e-12
    assert np.array_equal(o[0], v[0].astype(np.float64))       # row 0 sees only key 0


def test_prefill_rows_match_full_rows(oracle):
    T, D = 90, 128
    q = synth.normal_fp16((T, D), 27).numpy()
    k = synth.keys_fp16((T, D), 28).numpy()
    v = synth.normal_fp16((T, D), 29).numpy()
    rows = np.array([0, 1, 44, 89, 7])
    full = oracle.prefill_attention(q, k, v, TAU)
    assert np.array_equal(oracle.prefill_attention_rows(q, k, v, rows, TAU), full[rows])


def test_decode_advance_equals_step_bookkeeping(oracle):
    D, N = 128, 100
    k = synth.keys_fp16((N + 40, D), 71).numpy()
    v = synth.normal_fp16((N + 40, D), 72).numpy()
    q = synth.normal_fp16((1, D), 73).numpy()
    a = oracle.SliceCache.from_kept(k[:N], v[:N], R=32, G=32, Gv=128)
    b = oracle.SliceCache.from_kept(k[:N], v[:N], R=32, G=32, Gv=128)
    for i in range(40):
        a.step(q, k[N + i], v[N + i], TAU)
        b.advance(k[N + i], v[N + i])
    for key in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero"):
        assert np.array_equal(getattr(a, key), getattr(b, key))
    assert np.array_equal(np.array(a.res_k), np.array(b.res_k))


def test_prefill_attention_equal_keys_is_running_mean(oracle):
    T, D = 40, 128
    q = synth.normal_fp16((T, D), 24).numpy()
    k = np.tile(synth.keys_fp16((1, D), 25).numpy(), (T, 1))
    v = synth.normal_fp16((T, D), 26).numpy()
    o = oracle.prefill_attention(q, k, v, TAU)
    ref = np.cumsum(v.astype(np.float64), 0) / np.arange(1, T + 1)[:, None]
    assert np.max(np.abs(o - ref)) < 1e-12


# ------------------------------------------------------ O2 window scores

def test_window_scores_bruteforce_and_mass(oracle):
    for g, T, W in ((1, 48, 8), (4, 64, 32), (2, 33, 33), (3, 20, 1)):
        D = 128
        q = synth.normal_fp16((g, T, D), 31 + T).numpy()
        k = synth.keys_fp16((T, D), 32 + T).numpy()
        s = oracle.window_scores(q, k, W, TAU)
        qt = torch.from_numpy(q.astype(np.float64))
        kt = torch.from_numpy(k.astype(np.float64))
        logits = TAU * qt @ kt.T
        mask = torch.triu(torch.ones(T, T, dtype=torch.bool), 1)
        P = torch.softmax(logits.masked_fill(mask, -math.inf), -1)
        ref = P[:, T - W:, :].sum((0, 1)).numpy()
        assert np.max(np.abs(s - ref)) < 1e-12
        assert abs(s.sum() - W * g) < 1e-9
        assert np.all(s >= 0)


# --------------------------------------------------------------- O3 select

def _select_brute(s, W, keep):
    T = s.size
    if keep >= T:
        return np.arange(T)
    cand = np.arange(T - W)
    order = np.lexsort((cand, -s[: T - W]))         # score desc, then index asc
    return np.sort(np.concatenate([cand[order][: keep - W], np.arange(T - W, T)]))


def test_select_bruteforce_with_ties(oracle):
    rng = np.random.default_rng(6)
    for T in (1, 2, 17, 64, 300, 4096):
        for _ in range(4):
            W = int(rng.integers(0, min(T, 40) + 1))
            keep = int(rng.integers(W, T + 3))
            s = rng.integers(0, 6, T).astype(np.float64) / 7.0     # many exact ties
            got = oracle.select(s, W, keep)
            assert np.array_equal(got, _select_brute(s, W, keep))
            if keep < T:
                assert got.size == keep
    # a tie at the boundary goes to the lower index
    s = np.array([0.5, 0.9, 0.5, 0.5, 0.1, 0.0])
    assert list(oracle.select(s, 1, 3)) == [0, 1, 5]


def test_select_rejects_window_above_budget(oracle):
    with pytest.raises(ValueError):
        oracle.select(np.zeros(10), 5, 4)


# --------------------------------------------------------------- O9 decode

def _np_dequant(sc, G, Gv):
    """Independent dequant: numpy bit unpacking and numpy fp16 views."""
    D = sc.D
    kc, vc = _unpack(sc.k_codes, D).astype(np.float64), _unpack(sc.v_codes, D).astype(np.float64)
    ks = np.repeat(sc.k_scale.view(np.float16).astype(np.float64), G, 0)
    kz = np.repeat(sc.k_zero.view(np.float16).astype(np.float64), G, 0)
    vs = np.repeat(sc.v_scale.view(np.float16).astype(np.float64), Gv, 1)
    vz = np.repeat(sc.v_zero.view(np.float16).astype(np.float64), Gv, 1)
    return kc * ks + kz, vc * vs + vz


def _attend_ref(q, kk, vv):
    qt = torch.from_numpy(q.astype(np.float64))[None]          # [1, g, D]
    kt = torch.from_numpy(kk.astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(vv.astype(np.float64))[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt[:, :, None, :], kt, vt, scale=TAU)
    return o[0, :, 0, :].numpy()


def test_decode_full_precision_equals_dense(oracle):
    """Budget 100% and R above the length: no eviction, no quantization, so the
    decode step is plain attention over all tokens."""
    D, N, g = 128, 50, 4
    k = synth.keys_fp16((N, D), 41).numpy()
    v = synth.normal_fp16((N, D), 42).numpy()
    q = synth.normal_fp16((g, D), 43).numpy()
    kn = synth.keys_fp16((D,), 44).numpy()
    vn = synth.normal_fp16((D,), 45).numpy()
    sc = oracle.SliceCache.from_kept(k, v, R=128, G=32, Gv=128)
    assert sc.n_q == 0 and sc.r == N
    out = sc.step(q, kn, vn, TAU)
    ref = _attend_ref(q, np.vstack([k, kn[None]]), np.vstack([v, vn[None]]))
    assert np.max(np.abs(out - ref)) < 1e-12


def test_decode_quantized_equals_dense_over_dequant(oracle):
    D, N, g, G, Gv, R = 128, 300, 2, 32, 64, 32
    k = synth.keys_fp16((N, D), 51).numpy()
    v = synth.normal_fp16((N, D), 52).numpy()
    q = synth.normal_fp16((g, D), 53).numpy()
    kn = synth.keys_fp16((D,), 54).numpy()
    vn = synth.normal_fp16((D,), 55).numpy()
    sc = oracle.SliceCache.from_kept(k, v, R=R, G=G, Gv=Gv)
    nq, r = oracle.split(N, R, G)
    assert (sc.n_q, sc.r) == (nq, r)
    kh, vh = _np_dequant(sc, G, Gv)
    out = sc.step(q, kn, vn, TAU)
    kk = np.vstack([kh, k[nq:].astype(np.float64), kn[None].astype(np.float64)])
    vv = np.vstack([vh, v[nq:].astype(np.float64), vn[None].astype(np.float64)])
    assert np.max(np.abs(out - _attend_ref(q, kk, vv))) < 1e-12


def test_decode_flush_packs_oldest_group(oracle):
    """Appending until r reaches R+G packs exactly the oldest G residual tokens,
    the same codes as packing that stretch of the sequence directly."""
    D, G, Gv, R = 128, 32, 128, 32
    N = 64 + R + G - 2                               # r = R+G-2 after the split
    steps = 2 + G
    k = synth.keys_fp16((N + steps, D), 61).numpy()
    v = synth.normal_fp16((N + steps, D), 62).numpy()
    q = synth.normal_fp16((1, D), 63).numpy()
    sc = oracle.SliceCache.from_kept(k[:N], v[:N], R=R, G=G, Gv=Gv)
    assert (sc.n_q, sc.r) == (64, R + G - 2)
    sc.step(q, k[N], v[N], TAU)
    assert sc.n_q == 64 and sc.r == R + G - 1
    sc.step(q, k[N + 1], v[N + 1], TAU)              # r hits R+G -> flush
    assert sc.n_q == 64 + G and sc.r == R
    ref = oracle.pack_tokens(k[64:64 + G], v[64:64 + G], G, Gv)
    assert np.array_equal(sc.k_codes[64:], ref["k_codes"])
    assert np.array_equal(sc.k_scale[2:], ref["k_scale"])
    assert np.array_equal(sc.v_zero[64:], ref["v_zero"])
    for i in range(G):
        sc.step(q, k[N + 2 + i], v[N + 2 + i], TAU)
    assert sc.n_q == 64 + 2 * G and sc.r == R
    whole = oracle.pack_tokens(k[: 64 + 2 * G], v[: 64 + 2 * G], G, Gv)
    for key in whole:
        assert np.array_equal(getattr(sc, key), whole[key]), key


# ------------------------------------------------------ O10 decode mass

def test_decode_mass_matches_dense_softmax(oracle):
    """Per-token mass = softmax over the dequantized keys (independent numpy
    dequant, torch fp64 softmax) summed over the group's heads; it sums to g and
    the attention output is O9's."""
    D, N, g, G, Gv, R = 128, 300, 3, 32, 64, 32
    k = synth.keys_fp16((N, D), 71).numpy()
    v = synth.normal_fp16((N, D), 72).numpy()
    q = synth.normal_fp16((g, D), 73).numpy()
    kn = synth.keys_fp16((D,), 74).numpy()
    vn = synth.normal_fp16((D,), 75).numpy()
    sc = oracle.SliceCache.from_kept(k, v, R=R, G=G, Gv=Gv)
    twin = oracle.SliceCache.from_kept(k, v, R=R, G=G, Gv=Gv)
    nq = sc.n_q
    kh, _ = _np_dequant(sc, G, Gv)
    acc = np.zeros(N + 1)
    out = sc.step_mass(q, kn, vn, TAU, acc)
    kk = np.vstack([kh, k[nq:].astype(np.float64), kn[None].astype(np.float64)])
    logits = torch.from_numpy(q.astype(np.float64)) @ torch.from_numpy(kk).T * TAU
    ref = torch.softmax(logits, dim=-1).sum(0).numpy()
    assert np.max(np.abs(acc - ref)) < 1e-13
    assert abs(acc.sum() - g) < 1e-12
    assert np.array_equal(out, twin.step(q, kn, vn, TAU))


def test_decode_mass_single_head_weights_reproduce_output(oracle):
    """g = 1: the mass is the softmax weight vector, so sum_t mass_t nu_t is the
    O9 output (values dequantized independently)."""
    D, N, G, Gv, R = 128, 200, 32, 32, 32
    k = synth.keys_fp16((N, D), 81).numpy()
    v = synth.normal_fp16((N, D), 82).numpy()
    q = synth.normal_fp16((1, D), 83).numpy()
    sc = oracle.SliceCache.from_kept(k, v, R=R, G=G, Gv=Gv)
    nq = sc.n_q
    _, vh = _np_dequant(sc, G, Gv)
    out, mass = sc.attend_mass(q, TAU)
    vv = np.vstack([vh, v[nq:].astype(np.float64)])
    assert np.max(np.abs(mass @ vv - out[0])) < 1e-12


def test_decode_mass_zero_query_is_uniform(oracle):
    D, N, g = 128, 130, 4
    k = synth.keys_fp16((N, D), 91).numpy()
    v = synth.normal_fp16((N, D), 92).numpy()
    sc = oracle.SliceCache.from_kept(k, v, R=32, G=32, Gv=128)
    _, mass = sc.attend_mass(np.zeros((g, D), np.float16), TAU)
    assert mass.shape == (N,)
    assert np.max(np.abs(mass - g / N)) < 1e-15


def test_decode_mass_accumulates_by_arrival_order_across_flush(oracle):
    """Closed form.  Queries see only channel 0; every key has channel 0 = 0
    except one 'beacon' token appended at step s0 (channel 0 = 30, exact after
    2-bit packing: its group's channel-0 range is [0, 30], scale 10).  Before the
    beacon every step is uniform, g/n per token; from then on the beacon takes
    all but ~n e^-21 of every head's mass.  The beacon is flushed into the packed
    part midway and must keep its position."""
    D, G, Gv, R, g = 128, 32, 128, 32, 2
    N = 64 + R + G - 6                      # r = R+G-6 after the split
    steps, s0 = 12, 3                       # beacon at arrival position N+3; flush at step 5
    rng = np.random.default_rng(5)
    k = f16(rng.standard_normal((N + steps, D)))
    k[:, 0] = 0
    k[N + s0, 0] = 30
    v = f16(rng.standard_normal((N + steps, D)))
    q = np.zeros((g, D), np.float16)
    q[:, 0] = 8
    sc = oracle.SliceCache.from_kept(k[:N], v[:N], R=R, G=G, Gv=Gv)
    acc = np.zeros(N + steps)
    flushed = False
    for s in range(steps):
        nq = sc.n_q
        sc.step_mass(q, k[N + s], v[N + s], TAU, acc)
        flushed |= sc.n_q > nq
        if s == s0 + 1:
            assert not flushed
    assert flushed and sc.n_q > N + s0 - sc.r   # the beacon now sits in the packed part
    n_after = steps - s0
    # tokens that arrived before the beacon: the uniform steps, plus at most e^-21 each after it
    for t in range(N + s0):
        exp_t = sum(g / (N + s + 1) for s in range(max(0, t - N), s0))
        assert abs(acc[t] - exp_t) < g * n_after * math.exp(-21) * 1.01, t
    assert abs(acc[N + s0] - g * n_after) < g * n_after * (N + steps) * math.exp(-21)
    assert abs(acc.sum() - g * steps) < 1e-9
