"""Python binding of libminikv.so (ctypes).

Argument marshalling only: every step of the path runs in the CUDA library.
Torch supplies device memory and the stream.  The functions carry the names
of the C entry points without the ``minikv_`` prefix.  There is no CPU
fallback: if the library is missing or a tensor is not a contiguous CUDA
tensor of the right dtype, the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MINIKV_LIB points the binding at another build of the library
LIB_PATH = os.environ.get("MINIKV_LIB", os.path.join(_PKG, "libminikv.so"))
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "minikv.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA = 0, -1, -2, -3, -4
OP_SELECT_PREFILL, OP_TOPK_EVICT, OP_DECODE_ATTN, OP_DECODE_ATTN_MASS = 1, 2, 3, 4

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t


class CacheStruct(ctypes.Structure):
    """Mirror of ``minikv_cache`` in include/minikv.h."""
    _fields_ = [("B", _I), ("Hkv", _I), ("D", _I), ("G", _I), ("Gv", _I), ("R", _I), ("cap", _I),
                ("k_codes", _P), ("v_codes", _P), ("k_scale", _P), ("k_zero", _P),
                ("v_scale", _P), ("v_zero", _P), ("k_res", _P), ("v_res", _P),
                ("n_packed", _I), ("n_res", _I), ("res_start", _I), ("seq", _P), ("dseq", _P)]

MAX_RAGGED_SEQS = 256


_SIGS = {
    "minikv_cache_bytes": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "minikv_cache_bind": (_I, [ctypes.POINTER(CacheStruct), _P, _Z, _I, _I, _I, _I, _I, _I, _I]),
    "minikv_cache_set_ragged": (_I, [ctypes.POINTER(CacheStruct), _P]),
    "minikv_cache_set_device_state": (_I, [ctypes.POINTER(CacheStruct), _P, _P]),
    "minikv_quant_pack": (_I, [ctypes.POINTER(CacheStruct), _P, _P, _I, _P]),
    "minikv_quant_pack_seq": (_I, [ctypes.POINTER(CacheStruct), _I, _P, _P, _I, _P]),
    "minikv_evict_pack_seq": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, ctypes.POINTER(CacheStruct), _I, _P]),
    "minikv_select_prefill": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P, _Z, _P]),
    "minikv_select_prefill_status": (_I, [_P, _Z, _I, _I, _I, _P, ctypes.POINTER(ctypes.c_uint)]),
    "minikv_topk_evict": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _Z, _P]),
    "minikv_evict_pack": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, ctypes.POINTER(CacheStruct), _P]),
    "minikv_decode_attn": (_I, [ctypes.POINTER(CacheStruct), _P, _P, _P, _I, _F, _P, _P, _Z, _P]),
    "minikv_decode_attn_mass": (_I, [ctypes.POINTER(CacheStruct), _P, _P, _P, _I, _F, _P, _P, _P, _Z, _P]),
    "minikv_decode_attn_static": (_I, [ctypes.POINTER(CacheStruct), _P, _P, _P, _I, _F, _P, _P]),
    "minikv_set_deterministic": (_I, [_I]),
    "minikv_decode_plan": (_I, [ctypes.POINTER(CacheStruct), ctypes.POINTER(_I), ctypes.POINTER(_I), _P, _I]),
    "minikv_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I, _I]),
    "minikv_last_error_string": (ctypes.c_char_p, []),
}

_lib = None


class MiniKVError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"minikv error {code}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_quantized_evicted_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != OK:
        raise MiniKVError(rc, lib().minikv_last_error_string().decode())


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise TypeError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream, device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def workspace_size(op: int, B: int, Hq: int, Hkv: int, T: int, D: int = 128, W: int = 0) -> int:
    return int(lib().minikv_workspace_size(op, B, Hq, Hkv, T, D, W))


class MiniKVCache:
    """One layer's packed 2-bit cache in one device buffer, plus the
    zero-filled decode workspace (its arrival counters must start at zero)."""

    def __init__(self, B: int, Hkv: int, cap: int, *, D: int = 128, G: int = 32, Gv: int = 128, R: int = 128,
                 device="cuda", Hq: int | None = None, ws: torch.Tensor | None = None):
        L = lib()
        n = int(L.minikv_cache_bytes(B, Hkv, D, G, Gv, R, cap))
        if n == 0:
            raise MiniKVError(ERR_INVALID_ARG, f"bad cache shape B={B} Hkv={Hkv} D={D} G={G} Gv={Gv} R={R} cap={cap}")
        self.buf = torch.zeros(n + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self._off = (-base) % 256
        self.c = CacheStruct()
        _check(L.minikv_cache_bind(ctypes.byref(self.c), base + self._off, n, B, Hkv, D, G, Gv, R, cap))
        self.device = self.buf.device
        if ws is None:
            ws = torch.zeros(workspace_size(OP_DECODE_ATTN, B, Hq or Hkv, Hkv, cap + R + G, D),
                             dtype=torch.uint8, device=device)
        self.ws = ws
        self._seq = None
        self.dseq = None

    def set_ragged(self) -> "MiniKVCache":
        """Give every sequence its own length (per-sequence host state, all empty)."""
        self._seq = (ctypes.c_int * (3 * self.B))()
        _check(lib().minikv_cache_set_ragged(ctypes.byref(self.c), ctypes.cast(self._seq, _P)))
        return self

    def set_device_state(self, stream=None) -> "MiniKVCache":
        """Keep the per-sequence state in device memory (dseq [B, 4] int32:
        n_packed, n_res, res_start, status): decode steps then queue the same
        launches every step and can be captured in a CUDA graph."""
        self.dseq = torch.zeros((self.B, 4), dtype=torch.int32, device=self.device)
        _check(lib().minikv_cache_set_device_state(ctypes.byref(self.c), self.dseq.data_ptr(),
                                                   _stream(stream, self.device)))
        return self

    @property
    def ragged(self) -> bool:
        return self._seq is not None or self.dseq is not None

    def seq_state(self, b: int) -> tuple[int, int, int]:
        """(n_packed, n_res, res_start) of sequence b (any kind of batch; a
        device-resident state is read back, which synchronizes)."""
        if self.dseq is not None:
            return tuple(int(x) for x in self.dseq[b, :3].cpu())
        if self._seq is None:
            return self.n_packed, self.n_res, self.res_start
        return self._seq[3 * b], self._seq[3 * b + 1], self._seq[3 * b + 2]

    def status(self) -> list[int]:
        """Device-state mode: per-sequence status words (1 = a flush was refused at cap)."""
        return [int(x) for x in self.dseq[:, 3].cpu()] if self.dseq is not None else [0] * self.B

    # shape / state
    B = property(lambda s: s.c.B)
    Hkv = property(lambda s: s.c.Hkv)
    D = property(lambda s: s.c.D)
    G = property(lambda s: s.c.G)
    Gv = property(lambda s: s.c.Gv)
    R = property(lambda s: s.c.R)
    cap = property(lambda s: s.c.cap)
    n_packed = property(lambda s: s.c.n_packed)
    n_res = property(lambda s: s.c.n_res)
    res_start = property(lambda s: s.c.res_start)

    def _view(self, ptr: int, dtype: torch.dtype, shape) -> torch.Tensor:
        start = ptr - self.buf.data_ptr()
        nbytes = math.prod(shape) * torch.tensor([], dtype=dtype).element_size()
        return self.buf[start:start + nbytes].view(dtype).view(*shape)

    def arrays(self) -> dict:
        """Views of the device arrays (full capacity)."""
        B, H, D, G, Gv, cap = self.B, self.Hkv, self.D, self.G, self.Gv, self.cap
        ring = self.R + G
        return dict(
            k_codes=self._view(self.c.k_codes, torch.int32, (B, H, cap, D // 16)),
            v_codes=self._view(self.c.v_codes, torch.int32, (B, H, cap, D // 16)),
            k_scale=self._view(self.c.k_scale, torch.float16, (B, H, cap // G, D)),
            k_zero=self._view(self.c.k_zero, torch.float16, (B, H, cap // G, D)),
            v_scale=self._view(self.c.v_scale, torch.float16, (B, H, cap, D // Gv)),
            v_zero=self._view(self.c.v_zero, torch.float16, (B, H, cap, D // Gv)),
            k_res=self._view(self.c.k_res, torch.float16, (B, H, ring, D)),
            v_res=self._view(self.c.v_res, torch.float16, (B, H, ring, D)))

    def residual(self) -> tuple[torch.Tensor, torch.Tensor]:
        """Residual tokens in logical order (oldest first): [B, Hkv, n_res, D] (uniform batch)."""
        a = self.arrays()
        ring = self.R + self.G
        idx = torch.tensor([(self.res_start + i) % ring for i in range(self.n_res)], device=self.device,
                           dtype=torch.long)
        return a["k_res"][:, :, idx], a["v_res"][:, :, idx]

    def residual_seq(self, b: int) -> tuple[torch.Tensor, torch.Tensor]:
        """Residual tokens of sequence b in logical order: [Hkv, n_res_b, D]."""
        a = self.arrays()
        ring = self.R + self.G
        _, n_res, rs = self.seq_state(b)
        idx = torch.tensor([(rs + i) % ring for i in range(n_res)], device=self.device, dtype=torch.long)
        return a["k_res"][b][:, idx], a["v_res"][b][:, idx]

    def byte_counts(self) -> dict:
        """Algorithmic bytes the next decode step reads, per (b, KV head) of a
        uniform batch; on a ragged batch, summed over all units ('total')."""
        D, G, Gv = self.D, self.G, self.Gv

        def unit(nq, r):
            return nq * (D // 4) * 2 + (nq // G) * D * 4 + nq * (D // Gv) * 4, r * D * 4
        if not self.ragged:
            packed, res = unit(self.n_packed, self.n_res + 1)
            return dict(packed=packed, residual=res, per_unit=packed + res, total=(packed + res) * self.B * self.Hkv)
        st = [self.seq_state(b) for b in range(self.B)]
        tot = sum(sum(unit(nq, nr + 1)) for nq, nr, _ in st) * self.Hkv
        return dict(total=tot)


def quant_pack(cache: MiniKVCache, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
    """Load a compacted kept sequence k, v [B, Hkv, N, D] fp16 into the cache."""
    N = k.shape[2] if k.dim() == 4 else 0
    if k.shape != v.shape or k.shape[:2] != (cache.B, cache.Hkv) or k.shape[3] != cache.D:
        raise ValueError(f"k/v shape {tuple(k.shape)} does not match the cache")
    kp = _dev(k, torch.float16, "k") if N else None
    vp = _dev(v, torch.float16, "v") if N else None
    _check(lib().minikv_quant_pack(ctypes.byref(cache.c), kp, vp, N, _stream(stream, cache.device)))


def quant_pack_seq(cache: MiniKVCache, b: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
    """Load sequence b of a ragged cache: k, v [Hkv, N, D] fp16 (N of its own)."""
    N = k.shape[1] if k.dim() == 3 else 0
    if k.shape != v.shape or k.shape[0] != cache.Hkv or k.shape[2] != cache.D:
        raise ValueError(f"k/v shape {tuple(k.shape)} does not match the cache")
    kp = _dev(k, torch.float16, "k") if N else None
    vp = _dev(v, torch.float16, "v") if N else None
    _check(lib().minikv_quant_pack_seq(ctypes.byref(cache.c), b, kp, vp, N, _stream(stream, cache.device)))


def evict_pack_seq(cache: MiniKVCache, b: int, scores: torch.Tensor, k: torch.Tensor, v: torch.Tensor, W: int,
                   keep: int, idx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One prompt (scores [Hkv, T], k, v [Hkv, T, D]) kept and packed into
    sequence b of a ragged cache; returns idx [Hkv, min(keep, T)]."""
    Hkv, T, D = k.shape
    n = min(keep, T)
    if idx is None:
        idx = torch.empty((Hkv, n), dtype=torch.int32, device=k.device)
    _check(lib().minikv_evict_pack_seq(
        _dev(scores, torch.float32, "scores"), _dev(k, torch.float16, "k"), _dev(v, torch.float16, "v"),
        Hkv, T, D, W, keep, _dev(idx, torch.int32, "idx"), ctypes.byref(cache.c), b, _stream(stream, k.device)))
    return idx


def select_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, W: int, sm_scale: float | None = None,
                   o: torch.Tensor | None = None, scores: torch.Tensor | None = None,
                   ws: torch.Tensor | None = None, stream=None):
    """Causal attention output o [B, Hq, T, D] and window scores [B, Hkv, T] fp32."""
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if o is None:
        o = torch.empty_like(q)
    if scores is None:
        scores = torch.empty((B, Hkv, T), dtype=torch.float32, device=q.device)
    need = workspace_size(OP_SELECT_PREFILL, B, Hq, Hkv, T, D, W)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().minikv_select_prefill(
        _dev(q, torch.float16, "q"), _dev(k, torch.float16, "k"), _dev(v, torch.float16, "v"),
        B, Hq, Hkv, T, D, W, float(sm_scale), _dev(o, torch.float16, "o"),
        _dev(scores, torch.float32, "scores"), _dev(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream, q.device)))
    return o, scores


def select_prefill_status(ws: torch.Tensor, B: int, Hq: int, W: int, stream=None, library=None) -> int:
    """Status word of the last select_prefill on `ws` (synchronizes the stream):
    0 = finished, bit 0 = a bounded wait in the flash-attention pass expired."""
    st = ctypes.c_uint(0)
    L = library or lib()
    _check(L.minikv_select_prefill_status(_dev(ws, torch.uint8, "ws"), ws.numel(), B, Hq, W,
                                          _stream(stream, ws.device), ctypes.byref(st)))
    return int(st.value)


def topk_evict(scores: torch.Tensor, k: torch.Tensor, v: torch.Tensor, W: int, keep: int,
               idx: torch.Tensor | None = None, k_kept: torch.Tensor | None = None,
               v_kept: torch.Tensor | None = None, stream=None):
    """Kept positions idx [B, Hkv, n] (ascending) and the gathered rows."""
    B, Hkv, T, D = k.shape
    n = min(keep, T)
    if idx is None:
        idx = torch.empty((B, Hkv, n), dtype=torch.int32, device=k.device)
    if k_kept is None:
        k_kept = torch.empty((B, Hkv, n, D), dtype=torch.float16, device=k.device)
    if v_kept is None:
        v_kept = torch.empty((B, Hkv, n, D), dtype=torch.float16, device=k.device)
    _check(lib().minikv_topk_evict(
        _dev(scores, torch.float32, "scores"), _dev(k, torch.float16, "k"), _dev(v, torch.float16, "v"),
        B, Hkv, T, D, W, keep, _dev(idx, torch.int32, "idx"), _dev(k_kept, torch.float16, "k_kept"),
        _dev(v_kept, torch.float16, "v_kept"), None, 0, _stream(stream, k.device)))
    return idx, k_kept, v_kept


def evict_pack(cache: MiniKVCache, scores: torch.Tensor, k: torch.Tensor, v: torch.Tensor, W: int, keep: int,
               idx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """topk_evict + quant_pack in one call: the kept rows of the prompt k, v
    [B, Hkv, T, D] go straight into the cache; returns idx [B, Hkv, n]."""
    B, Hkv, T, D = k.shape
    n = min(keep, T)
    if idx is None:
        idx = torch.empty((B, Hkv, n), dtype=torch.int32, device=k.device)
    _check(lib().minikv_evict_pack(
        _dev(scores, torch.float32, "scores"), _dev(k, torch.float16, "k"), _dev(v, torch.float16, "v"),
        B, Hkv, T, D, W, keep, _dev(idx, torch.int32, "idx"), ctypes.byref(cache.c), _stream(stream, k.device)))
    return idx


def decode_attn(cache: MiniKVCache, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                sm_scale: float | None = None, out: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One decode step: q [B, Hq, D], k_new/v_new [B, Hkv, D] -> out [B, Hq, D]."""
    B, Hq, D = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if ws is None:
        ws = cache.ws
    _check(lib().minikv_decode_attn(
        ctypes.byref(cache.c), _dev(q, torch.float16, "q"), _dev(k_new, torch.float16, "k_new"),
        _dev(v_new, torch.float16, "v_new"), Hq, float(sm_scale), _dev(out, torch.float16, "out"),
        _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream, q.device)))
    return out


def decode_attn_mass(cache: MiniKVCache, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                     mass: torch.Tensor, sm_scale: float | None = None, out: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """decode_attn that also adds this step's attention mass of every cached
    token into mass [B, Hkv, cap + R + G] fp32 (tokens in arrival order).  The
    default workspace is made once per cache, zero-filled, and kept on it."""
    B, Hq, D = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if tuple(mass.shape) != (cache.B, cache.Hkv, cache.cap + cache.R + cache.G):
        raise ValueError(f"mass shape {tuple(mass.shape)}: expected {(cache.B, cache.Hkv, cache.cap + cache.R + cache.G)}")
    if ws is None:
        need = workspace_size(OP_DECODE_ATTN_MASS, B, Hq, cache.Hkv, cache.cap + cache.R + cache.G, D)
        if getattr(cache, "ws_mass", None) is None or cache.ws_mass.numel() < need:
            cache.ws_mass = torch.zeros(need, dtype=torch.uint8, device=cache.device)
        ws = cache.ws_mass
    _check(lib().minikv_decode_attn_mass(
        ctypes.byref(cache.c), _dev(q, torch.float16, "q"), _dev(k_new, torch.float16, "k_new"),
        _dev(v_new, torch.float16, "v_new"), Hq, float(sm_scale), _dev(out, torch.float16, "out"),
        _dev(mass, torch.float32, "mass"), _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream, q.device)))
    return out


def decode_plan(cache) -> tuple:
    """(CTAs, boundary weight, first item of each CTA's range + the item count)
    of the next decode call on `cache` (a MiniKVCache or a bound CacheStruct);
    host logic only.  The list is empty for a device-resident state."""
    c = cache.c if hasattr(cache, "c") else cache
    ctas, wu = _I(0), _I(0)
    _check(lib().minikv_decode_plan(ctypes.byref(c), ctypes.byref(ctas), ctypes.byref(wu), None, 0))
    if c.dseq:
        return ctas.value, wu.value, []
    first = (_I * (ctas.value + 1))()
    _check(lib().minikv_decode_plan(ctypes.byref(c), ctypes.byref(ctas), ctypes.byref(wu), first, ctas.value + 1))
    return ctas.value, wu.value, list(first)


def set_deterministic(on: bool) -> None:
    """Fixed assignment of decode items to warps (bit-identical repeat calls)
    instead of dynamic claiming (the default); process-wide."""
    _check(lib().minikv_set_deterministic(1 if on else 0))


def decode_attn_static(cache: MiniKVCache, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                       sm_scale: float | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """decode_attn for callers that may not allocate device memory: the split
    partials live in the library's own fixed 8 MiB device array instead of a
    workspace (no cudaMalloc anywhere in the call).  Calls whose GPU work
    overlaps share that array and race on it."""
    B, Hq, D = q.shape
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    _check(lib().minikv_decode_attn_static(
        ctypes.byref(cache.c), _dev(q, torch.float16, "q"), _dev(k_new, torch.float16, "k_new"),
        _dev(v_new, torch.float16, "v_new"), Hq, float(sm_scale), _dev(out, torch.float16, "out"),
        _stream(stream, q.device)))
    return out
