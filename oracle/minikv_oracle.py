"""MiniKV CPU oracle: Python side.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product library never calls it and
shares nothing with it: the arithmetic lives in ``minikv_oracle.c`` next to
this file (built with gcc, no FMA contraction, IEEE fp32/fp64), and this module
only marshals numpy arrays into it and keeps the per-slice decode state
(append, attend, flush), which is plain list bookkeeping.

Step names O1..O9 follow the restatement in ``minikv_oracle.c``:
  O1 prefill attention        O2 observation-window scores   O3 select
  O4 gather                   O5 split                       O6 quantize
  O7 bit packing              O8 dequant                     O9 decode step
  O10 decode-time attention mass (H2O-style accumulated score)
Sources: the MiniKV abstract (2-bit layer-discriminative KV cache, kernels
compatible with FlashAttention) and the gptget.net summary of arXiv 2411.18077,
sections 方法论 / 方法详解 (sub-channel key quantization, per-token value
quantization, selective flash attention by a second kernel, importance-based
adaptive KV) and 实验设计 (H2O, the accumulated-attention eviction MiniKV is
compared with).

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against fp16 library rounding (numpy), torch fp64 attention, closed forms,
invariants and brute force.  None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "minikv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libminikv_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile minikv_oracle.c into libminikv_oracle.so (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_long
_D = ctypes.c_double

_SIGS = {
    "oracle_half_to_double": (_D, [ctypes.c_uint16]),
    "oracle_float_to_half": (ctypes.c_uint16, [ctypes.c_float]),
    "oracle_split": (None, [_I, _I, _I, _P, _P]),
    "oracle_quantize_group": (None, [_P, _I, _L, _P, _P, _P]),
    "oracle_pack_token": (None, [_P, _I, _P]),
    "oracle_pack_tokens": (None, [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]),
    "oracle_dequant_tokens": (None, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "oracle_prefill_attention": (None, [_P, _P, _P, _I, _I, _D, _P]),
    "oracle_prefill_attention_rows": (None, [_P, _P, _P, _I, _I, _D, _P, _I, _P]),
    "oracle_window_scores": (None, [_P, _P, _I, _I, _I, _I, _D, _P]),
    "oracle_select": (_I, [_P, _I, _I, _I, _P]),
    "oracle_decode_attention": (None, [_P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _D, _P]),
    "oracle_decode_attention_mass": (None, [_P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _D, _P,
                                            _P]),
}


def lib():
    global _lib
    if _lib is None:
        path = build_oracle()
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _h(a) -> np.ndarray:
    """fp16 array (any float16 / uint16 array-like) -> contiguous uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return np.ascontiguousarray(a)


# ------------------------------------------------------------------ fp16

def half_to_double(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = lib().oracle_half_to_double
    return np.array([f(int(x)) for x in b], dtype=np.float64)


def float_to_half(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float32).ravel()
    f = lib().oracle_float_to_half
    return np.array([f(float(v)) for v in a], dtype=np.uint16)


# ------------------------------------------------------ O5, O6, O7, O8

def split(N: int, R: int, G: int) -> tuple[int, int]:
    """O5: N kept tokens -> (n_q packed, r residual)."""
    nq, r = ctypes.c_int(), ctypes.c_int()
    lib().oracle_split(N, R, G, ctypes.byref(nq), ctypes.byref(r))
    return nq.value, r.value


def quantize_group(x) -> tuple[int, int, np.ndarray]:
    """O6 on one group of fp16 values -> (scale bits, zero bits, codes uint8)."""
    xb = _h(x).ravel()
    s, z = ctypes.c_uint16(), ctypes.c_uint16()
    codes = np.zeros(xb.size, np.uint8)
    lib().oracle_quantize_group(_ptr(xb), xb.size, 1, ctypes.byref(s), ctypes.byref(z), _ptr(codes))
    return s.value, z.value, codes


def pack_token(codes) -> np.ndarray:
    """O7: one token's D codes -> D/16 uint32 words."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    w = np.zeros(c.size // 16, np.uint32)
    lib().oracle_pack_token(_ptr(c), c.size, _ptr(w))
    return w


def pack_tokens(k, v, G: int, Gv: int) -> dict:
    """O5-O7 for one (b, kv-head) slice whose n_q tokens (multiple of G) are all packed."""
    kb, vb = _h(k), _h(v)
    n_q, D = kb.shape
    assert n_q % G == 0 and D % 16 == 0 and D % Gv == 0
    out = dict(
        k_codes=np.zeros((n_q, D // 16), np.uint32), k_scale=np.zeros((n_q // G, D), np.uint16),
        k_zero=np.zeros((n_q // G, D), np.uint16), v_codes=np.zeros((n_q, D // 16), np.uint32),
        v_scale=np.zeros((n_q, D // Gv), np.uint16), v_zero=np.zeros((n_q, D // Gv), np.uint16))
    lib().oracle_pack_tokens(_ptr(kb), _ptr(vb), n_q, D, G, Gv,
                             _ptr(out["k_codes"]), _ptr(out["k_scale"]), _ptr(out["k_zero"]),
                             _ptr(out["v_codes"]), _ptr(out["v_scale"]), _ptr(out["v_zero"]))
    return out


def dequant_tokens(p: dict, G: int, Gv: int) -> tuple[np.ndarray, np.ndarray]:
    """O8: packed slice -> fp64 (k_hat, v_hat) [n_q, D]."""
    n_q, D = p["k_codes"].shape[0], p["k_codes"].shape[1] * 16
    kh = np.zeros((n_q, D)); vh = np.zeros((n_q, D))
    a = {k: np.ascontiguousarray(p[k]) for k in ("k_codes", "k_scale", "k_zero", "v_codes", "v_scale", "v_zero")}
    lib().oracle_dequant_tokens(_ptr(a["k_codes"]), _ptr(a["k_scale"]), _ptr(a["k_zero"]),
                                _ptr(a["v_codes"]), _ptr(a["v_scale"]), _ptr(a["v_zero"]),
                                n_q, D, G, Gv, _ptr(kh), _ptr(vh))
    return kh, vh


# ------------------------------------------------------------ O1, O2, O3, O4

def prefill_attention(q, k, v, tau: float) -> np.ndarray:
    """O1 for one query head: q, k, v [T, D] fp16 -> o [T, D] fp64 (causal)."""
    qb, kb, vb = _h(q), _h(k), _h(v)
    T, D = qb.shape
    o = np.zeros((T, D))
    lib().oracle_prefill_attention(_ptr(qb), _ptr(kb), _ptr(vb), T, D, tau, _ptr(o))
    return o


def prefill_attention_rows(q, k, v, rows, tau: float) -> np.ndarray:
    """O1 for the listed query rows of one head: -> [len(rows), D] fp64."""
    qb, kb, vb = _h(q), _h(k), _h(v)
    T, D = qb.shape
    r = np.ascontiguousarray(rows, dtype=np.int32)
    out = np.zeros((r.size, D))
    lib().oracle_prefill_attention_rows(_ptr(qb), _ptr(kb), _ptr(vb), T, D, tau, _ptr(r), r.size, _ptr(out))
    return out


def window_scores(q_group, k, W: int, tau: float) -> np.ndarray:
    """O2 for one KV head: q_group [g, T, D], k [T, D] fp16 -> s [T] fp64."""
    qb, kb = _h(q_group), _h(k)
    g, T, D = qb.shape
    s = np.zeros(T)
    lib().oracle_window_scores(_ptr(qb), _ptr(kb), g, T, D, W, tau, _ptr(s))
    return s


def select(s, W: int, keep: int) -> np.ndarray:
    """O3: scores [T] -> ascending kept positions (int32).  fp32 scores are
    widened to fp64 exactly, so the order they define is unchanged."""
    sd = np.ascontiguousarray(s, dtype=np.float64)
    T = sd.size
    idx = np.zeros(max(min(keep, T), 1), np.int32)
    n = lib().oracle_select(_ptr(sd), T, W, keep, _ptr(idx))
    if n < 0:
        raise ValueError("oracle_select: bad arguments")
    return idx[:n]


def gather(x, idx) -> np.ndarray:
    """O4: exact row copy x[idx]."""
    return np.ascontiguousarray(np.asarray(x)[np.asarray(idx)])


# ------------------------------------------------------------------ O9 decode

@dataclass
class SliceCache:
    """Decode state of one (b, kv-head) slice: packed tokens plus the fp16
    residual (oldest first).  Pure bookkeeping; arithmetic is in C."""
    D: int
    G: int
    Gv: int
    R: int
    k_codes: np.ndarray
    k_scale: np.ndarray
    k_zero: np.ndarray
    v_codes: np.ndarray
    v_scale: np.ndarray
    v_zero: np.ndarray
    res_k: list = field(default_factory=list)
    res_v: list = field(default_factory=list)

    @property
    def n_q(self) -> int:
        return self.k_codes.shape[0]

    @property
    def r(self) -> int:
        return len(self.res_k)

    @classmethod
    def from_kept(cls, k, v, R: int, G: int, Gv: int) -> "SliceCache":
        """O5-O7: load a compacted kept sequence [N, D]."""
        kb, vb = _h(k), _h(v)
        N, D = kb.shape
        n_q, r = split(N, R, G)
        p = pack_tokens(kb[:n_q], vb[:n_q], G, Gv)
        return cls(D, G, Gv, R, p["k_codes"], p["k_scale"], p["k_zero"], p["v_codes"],
                   p["v_scale"], p["v_zero"], [kb[n_q + i].copy() for i in range(r)],
                   [vb[n_q + i].copy() for i in range(r)])

    def attend(self, q, tau: float) -> np.ndarray:
        """O9 step 2: q [g, D] fp16 -> out [g, D] fp64 over packed + residual."""
        qb = _h(q)
        g = qb.shape[0]
        rk = np.ascontiguousarray(np.array(self.res_k, np.uint16).reshape(self.r, self.D))
        rv = np.ascontiguousarray(np.array(self.res_v, np.uint16).reshape(self.r, self.D))
        out = np.zeros((g, self.D))
        a = [np.ascontiguousarray(x) for x in (self.k_codes, self.k_scale, self.k_zero,
                                               self.v_codes, self.v_scale, self.v_zero)]
        lib().oracle_decode_attention(_ptr(qb), g, *(_ptr(x) for x in a), self.n_q,
                                      _ptr(rk), _ptr(rv), self.r, self.D, self.G, self.Gv,
                                      tau, _ptr(out))
        return out

    def attend_mass(self, q, tau: float) -> tuple[np.ndarray, np.ndarray]:
        """O9 + O10 step 2: q [g, D] fp16 -> (out [g, D], mass [n_q + r]) fp64.
        mass[t] = sum over the g heads of token t's softmax probability; t runs
        over the packed tokens, then the residual oldest first, i.e. the order in
        which the tokens entered this slice."""
        qb = _h(q)
        g = qb.shape[0]
        rk = np.ascontiguousarray(np.array(self.res_k, np.uint16).reshape(self.r, self.D))
        rv = np.ascontiguousarray(np.array(self.res_v, np.uint16).reshape(self.r, self.D))
        out = np.zeros((g, self.D))
        mass = np.zeros(self.n_q + self.r)
        a = [np.ascontiguousarray(x) for x in (self.k_codes, self.k_scale, self.k_zero,
                                               self.v_codes, self.v_scale, self.v_zero)]
        lib().oracle_decode_attention_mass(_ptr(qb), g, *(_ptr(x) for x in a), self.n_q,
                                           _ptr(rk), _ptr(rv), self.r, self.D, self.G, self.Gv,
                                           tau, _ptr(out), _ptr(mass))
        return out, mass

    def step_mass(self, q, k_new, v_new, tau: float, acc: np.ndarray) -> np.ndarray:
        """O9 + O10: append the new token, attend, add this step's mass to the
        running score acc[:n_q + r] (indexed by arrival order, which a flush
        keeps), then flush if due.  Returns out [g, D]."""
        self.res_k.append(_h(k_new).ravel().copy())
        self.res_v.append(_h(v_new).ravel().copy())
        out, mass = self.attend_mass(q, tau)
        acc[: mass.size] += mass
        if self.r == self.R + self.G:
            self.flush()
        return out

    def step(self, q, k_new, v_new, tau: float) -> np.ndarray:
        """O9: append the new token, attend, then flush G tokens if r == R+G."""
        self.res_k.append(_h(k_new).ravel().copy())
        self.res_v.append(_h(v_new).ravel().copy())
        out = self.attend(q, tau)
        if self.r == self.R + self.G:
            self.flush()
        return out

    def advance(self, k_new, v_new) -> None:
        """O9 without the attention: append the new token and flush if due
        (bookkeeping for steps whose output is not checked)."""
        self.res_k.append(_h(k_new).ravel().copy())
        self.res_v.append(_h(v_new).ravel().copy())
        if self.r == self.R + self.G:
            self.flush()

    def flush(self) -> None:
        """Pack the oldest G residual tokens as the next key group and G value tokens."""
        kb = np.array(self.res_k[: self.G], np.uint16)
        vb = np.array(self.res_v[: self.G], np.uint16)
        p = pack_tokens(kb, vb, self.G, self.Gv)
        self.k_codes = np.concatenate([self.k_codes, p["k_codes"]])
        self.k_scale = np.concatenate([self.k_scale, p["k_scale"]])
        self.k_zero = np.concatenate([self.k_zero, p["k_zero"]])
        self.v_codes = np.concatenate([self.v_codes, p["v_codes"]])
        self.v_scale = np.concatenate([self.v_scale, p["v_scale"]])
        self.v_zero = np.concatenate([self.v_zero, p["v_zero"]])
        del self.res_k[: self.G]
        del self.res_v[: self.G]


def pyramid_keep(T: int, layer: int, n_layers: int, p0_pct: int = 30, p1_pct: int = 5) -> int:
    """Per-layer keep count of a linear keep-fraction schedule (layer-discriminative
    budget, the MiniKV Pyramid rows of the LongBench table): fraction p0 at layer 0
    falling linearly to p1 at the last layer, k = floor(p * T) in integers."""
    num = p0_pct * (n_layers - 1) - (p0_pct - p1_pct) * layer
    return (T * num) // (100 * (n_layers - 1))
