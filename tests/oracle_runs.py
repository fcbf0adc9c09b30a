"""Drive the CPU oracle over batched [B, H, ...] tensors (test helper)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import minikv_oracle as O


def np16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy()


def pack_reference(k: torch.Tensor, v: torch.Tensor, R: int, G: int, Gv: int):
    """SliceCache per (b, h) for a kept sequence [B, H, N, D]."""
    kn, vn = np16(k), np16(v)
    B, H = kn.shape[:2]
    return [[O.SliceCache.from_kept(kn[b, h], vn[b, h], R, G, Gv) for h in range(H)] for b in range(B)]


def compare_cache(cache, ref, check_residual=True):
    """Bit-exact comparison of the GPU cache arrays with the oracle slices."""
    a = {k: v.cpu().numpy() for k, v in cache.arrays().items()}
    kr, vr = cache.residual()
    kr, vr = kr.cpu().numpy(), vr.cpu().numpy()
    B, H = cache.B, cache.Hkv
    G = cache.G
    for b in range(B):
        for h in range(H):
            s = ref[b][h]
            nq = s.n_q
            assert cache.n_packed == nq, (cache.n_packed, nq)
            assert cache.n_res == s.r, (cache.n_res, s.r)
            np.testing.assert_array_equal(a["k_codes"][b, h, :nq].view(np.uint32), s.k_codes)
            np.testing.assert_array_equal(a["v_codes"][b, h, :nq].view(np.uint32), s.v_codes)
            np.testing.assert_array_equal(a["k_scale"][b, h, :nq // G].view(np.uint16), s.k_scale)
            np.testing.assert_array_equal(a["k_zero"][b, h, :nq // G].view(np.uint16), s.k_zero)
            np.testing.assert_array_equal(a["v_scale"][b, h, :nq].view(np.uint16), s.v_scale)
            np.testing.assert_array_equal(a["v_zero"][b, h, :nq].view(np.uint16), s.v_zero)
            if check_residual:
                np.testing.assert_array_equal(kr[b, h].view(np.uint16), np.array(s.res_k, np.uint16).reshape(s.r, s.D))
                np.testing.assert_array_equal(vr[b, h].view(np.uint16), np.array(s.res_v, np.uint16).reshape(s.r, s.D))


def decode_reference_step(ref, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, tau: float) -> np.ndarray:
    """O9 on every (b, KV head): returns out [B, Hq, D] fp64 and advances ref."""
    qn, kn, vn = np16(q), np16(k_new), np16(v_new)
    B, Hq, D = qn.shape
    H = kn.shape[1]
    g = Hq // H
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(H):
            out[b, h * g:(h + 1) * g] = ref[b][h].step(qn[b, h * g:(h + 1) * g], kn[b, h], vn[b, h], tau)
    return out


def decode_mass_reference_step(ref, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, tau: float,
                               acc: np.ndarray) -> np.ndarray:
    """O9 + O10 on every (b, KV head): returns out [B, Hq, D] fp64, adds the
    step's mass into acc [B, Hkv, >= n] and advances ref."""
    qn, kn, vn = np16(q), np16(k_new), np16(v_new)
    B, Hq, D = qn.shape
    H = kn.shape[1]
    g = Hq // H
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(H):
            out[b, h * g:(h + 1) * g] = ref[b][h].step_mass(qn[b, h * g:(h + 1) * g], kn[b, h], vn[b, h], tau,
                                                            acc[b, h])
    return out


def prefill_reference(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, W: int, tau: float, heads=None):
    """O1 outputs for the listed (b, h) query heads and O2 scores for every (b, KV head)."""
    qn, kn, vn = np16(q), np16(k), np16(v)
    B, Hq, T, D = qn.shape
    H = kn.shape[1]
    g = Hq // H
    outs = {}
    for (b, h) in (heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]):
        outs[(b, h)] = O.prefill_attention(qn[b, h], kn[b, h // g], vn[b, h // g], tau)
    scores = np.zeros((B, H, T))
    for b in range(B):
        for h in range(H):
            scores[b, h] = O.window_scores(qn[b, h * g:(h + 1) * g], kn[b, h], W, tau)
    return outs, scores
