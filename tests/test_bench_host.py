"""Host-side accounting of bench.py, checked on CPU against the oracle's own
bookkeeping: the per-sequence lengths it mirrors step by step (they give the
algorithmic bytes behind the roofline figure) and its keep budgets."""
import numpy as np

import bench
from bit_quantized_evicted_b200 import synth


def test_length_mirror_follows_the_oracle_cache_through_flushes():
    G, R, D = 32, 32, 128
    lengths = [0, 5, 31, 32, 33, 64 + 40, 300]
    steps = 3 * G + 7
    mirror = bench.LengthMirror([lengths], G, R)
    slices = []
    for i, N in enumerate(lengths):
        k = synth.keys_fp16((max(N, 1), D), 1000 + i).numpy()[:N]
        v = synth.normal_fp16((max(N, 1), D), 2000 + i).numpy()[:N]
        slices.append(bench_oracle().SliceCache.from_kept(k, v, R, G, D))
    kn = synth.keys_fp16((D,), 7).numpy()
    vn = synth.normal_fp16((D,), 8).numpy()
    for s in range(steps):
        for (nq, nr), sl in zip(mirror.st[0], slices):
            assert (nq, nr) == (sl.n_q, sl.r), s
        # bytes of this step: every unit reads its packed tokens and its residual plus the new token
        expect = sum(84 * sl.n_q + 512 * (sl.r + 1) for sl in slices) * 8
        assert mirror.layer_bytes(0, 8, False) == expect
        assert mirror.layer_bytes(0, 8, True) == expect + sum(8 * (sl.n_q + sl.r + 1) for sl in slices) * 8
        mirror.advance()
        for sl in slices:
            sl.advance(kn, vn)


def bench_oracle():
    from oracle import minikv_oracle as O
    return O


def test_keep_budgets_match_the_oracle_schedule():
    O = bench_oracle()
    for T in (4096, 32768, 44000):
        for layer in range(32):
            assert bench.keep_of(T, "pyramid", layer, 32) == O.pyramid_keep(T, layer, 32)
        assert bench.keep_of(T, 20) == T * 20 // 100
    ragged = bench.DECODE_PRESETS["mistral7b_gqa_ragged_decode"]
    ctx = np.array(ragged["contexts"])
    assert ctx[0] == 4096 and ctx[-1] == 32768 and np.all(np.diff(ctx) > 0)
