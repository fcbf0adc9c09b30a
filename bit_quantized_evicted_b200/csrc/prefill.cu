// minikv_select_prefill: causal flash attention over the prompt plus the
// observation-window score pass.
//
// Source: gptget.net summary of arXiv 2411.18077, 方法详解 third bullet:
// "selective flash attention" implemented with a second kernel; MiniKV
// abstract: kernels compatible with FlashAttention.  Reading: the first kernel
// is an ordinary causal FlashAttention forward that also keeps the row
// log-sum-exp of the last W query rows; the second kernel recomputes those rows'
// probabilities P[i, j] = exp(s_ij - lse_i) and sums them per key over the rows
// and over the query heads of each KV head.
//
// Kernel 1 (fa_tc_kernel): one CTA per 128-row query tile of one (sequence,
// query head); S = Q K^T and O += P V on the tcgen05 tensor cores with fp32
// accumulators in tensor memory, Q/K/V brought in by TMA (128-byte swizzle),
// warp-specialised K and V producers, a single MMA-issuing thread and four
// softmax warps (one thread per query row).  Kernel 2 (window_score_kernel):
// one CTA per 64 keys of one KV head; S^T = K Q_w^T with mma.sync, then the
// column sums of exp(S - lse) over the window rows.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace minikv {

namespace {

constexpr int kBN = 64;   // keys per window-score CTA

// element offset of (row, col) in a [rows][128] fp16 tile, 16-byte chunks
// XOR-swizzled by row so ldmatrix row reads hit distinct banks
__device__ __forceinline__ int swz(int row, int col) {
    return row * kD + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7);
}

// copy `rows` rows (row0.., of a [T][128] fp16 matrix) into a swizzled tile;
// rows >= T are zero-filled
__device__ __forceinline__ void load_tile(uint16_t *tile, const uint16_t *g, int row0, int rows, int T) {
    for (int e = threadIdx.x; e < rows * 16; e += blockDim.x) {
        const int r = e >> 4, ch = e & 15;
        const int gr = row0 + r;
        const bool ok = gr < T;
        const uint16_t *src = g + (size_t)(ok ? gr : 0) * kD + ch * 8;
        cp_async16(smem_addr(tile + swz(r, ch * 8)), src, ok);
    }
}

// ---------------------------------------------------------------- kernel 1
//
// One CTA = one 128-row query tile of one (sequence, query head); 7 warps:
//   warp 0      TMA producer of the Q tile, then K_j into 3 stages;
//   warp 1      TMEM owner and the single thread issuing tcgen05.mma;
//   warp 2      TMA producer of V_j into 2 stages;
//   warps 3..6  softmax: thread = query row = TMEM lane (warp w reads lanes
//               32*(w%4) .. +31), plus the O rescale and the epilogue.
// Tensor memory (512 columns): S_0, S_1 fp32 [128 x 128] at 0 / 128; O fp32 at
// 256; P_0, P_1 (fp16 pairs, the A operand of P V) at 384 / 448.
// Issue order S_0, S_1, then (PV_j interleaved with S_{j+2}) as soon as P_j
// is written.  MMAs into one accumulator wait for each other (about 200 cycles
// each on B200), so two independent chains in flight roughly double the
// tensor-pipe throughput; meanwhile the softmax warps work on S_{j+1}.
// The running max is lazy: a row's reference max moves only when a new score
// exceeds it by more than 2^8 (p <= 256 stays exact enough in fp16), so O is
// rescaled rarely; l and O always refer to the same reference.
constexpr int kTileM = 128, kTileN = 128;
constexpr int kKStages = 3, kVStages = 2;
constexpr int kFaThreads = 224;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr float kLazyMax = 8.f;

struct FaSmem {
    uint16_t q[2][kTileM * 64];        // K-blocks of 64 fp16, 128-byte swizzle
    uint16_t k[kKStages][2][kTileN * 64];   // [stage][K-block]
    uint16_t v[kVStages][2][kTileN * 64];   // [stage][64-wide d block]: MN-major B of P V
    uint64_t q_full, k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t drain;   // the MMA issuer's last commit, waited on before tensor memory is freed
    uint32_t tmem_base;
    int abort;
};

struct FaArgs {
    float *lse2;        // [B, Hq, W] window rows, log2 domain
    unsigned *status;   // bit 0: a bounded wait expired in some CTA (its outputs are not valid)
    int Hq, Hkv, T, W, nqt;
    int hg;             // (sequence, head) pairs per scheduling group
    float scale_log2;
};

// Polls of an mbarrier before a wait of the pipeline gives up (seconds at the
// default).  A build with a tiny limit makes the waits run out while the copies
// and MMAs they wait for are still in flight: the abort path below then drains
// them and the status word reports the expiry.
#ifndef MINIKV_WAIT_LIMIT
#define MINIKV_WAIT_LIMIT (1u << 26)
#endif

// Bounded wait shared by a CTA: once any wait times out, every later wait
// returns false at once so all roles reach the final barrier.
__device__ __forceinline__ bool fa_wait(FaSmem &s, uint64_t *bar, uint32_t parity) {
    if (*reinterpret_cast<volatile int *>(&s.abort)) return false;
    if (mbar_wait(bar, parity, MINIKV_WAIT_LIMIT)) return true;
    *reinterpret_cast<volatile int *>(&s.abort) = 1;
    return false;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(kFaThreads, 1)
    fa_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_o, const FaArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    FaSmem &s = *reinterpret_cast<FaSmem *>(smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Groups of hg (sequence, head) pairs whose K / V fit in L2 together; inside
    // a group, query tiles heaviest first across all its heads, so the longest
    // CTAs start early and the last wave holds only short ones.
    const int BH = gridDim.x / a.nqt;
    const int grp = (int)blockIdx.x / (a.hg * a.nqt), rr = (int)blockIdx.x - grp * a.hg * a.nqt;
    const int ng = min(a.hg, BH - grp * a.hg);
    const int bh = grp * a.hg + rr % ng;
    const int qt = a.nqt - 1 - rr / ng;
    const int b = bh / a.Hq, h = bh % a.Hq;
    const int kvh = b * a.Hkv + h / (a.Hq / a.Hkv);
    const int nkb = qt + 1;   // causal: key blocks 0..qt

    if (tid == 0) {
        mbar_init(&s.q_full, 1);
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&s.k_full[i], 1);
            mbar_init(&s.k_empty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&s.v_full[i], 1);
            mbar_init(&s.v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.s_full[i], 1);
            mbar_init(&s.p_full[i], 128);
            mbar_init(&s.o_done[i], 1);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tc::tmem_alloc(&s.tmem_base, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            tc::prefetch_map(&map_q);
            tc::prefetch_map(&map_k);
            tc::prefetch_map(&map_v);
            mbar_arrive_expect_tx(&s.q_full, 2 * kTileM * 128);
            tc::tma_load_3d(s.q[0], &map_q, 0, qt * kTileM, bh, &s.q_full);
            tc::tma_load_3d(s.q[1], &map_q, 64, qt * kTileM, bh, &s.q_full);
            int issued = 0;
            for (int j = 0; j < nkb; ++j) {
                const int ks = j % kKStages;
                if (j >= kKStages && !fa_wait(s, &s.k_empty[ks], (j / kKStages - 1) & 1)) break;
                mbar_arrive_expect_tx(&s.k_full[ks], 2 * kTileN * 128);
                tc::tma_load_3d(s.k[ks][0], &map_k, 0, j * kTileN, kvh, &s.k_full[ks]);
                tc::tma_load_3d(s.k[ks][1], &map_k, 64, j * kTileN, kvh, &s.k_full[ks]);
                issued = j + 1;
            }
            if (*reinterpret_cast<volatile int *>(&s.abort)) {
                // a wait gave up: let the loads this thread queued land before the CTA exits
                // (each stage holds at most one unconsumed load; waits on a finished phase return at once)
                mbar_wait(&s.q_full, 0);
                for (int j = issued > kKStages ? issued - kKStages : 0; j < issued; ++j)
                    mbar_wait(&s.k_full[j % kKStages], (j / kKStages) & 1);
            }
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- V producer (its own thread: a V slot frees later than a K slot)
        if (lane == 0) {
            int issued = 0;
            for (int j = 0; j < nkb; ++j) {
                const int vs = j % kVStages;
                if (j >= kVStages && !fa_wait(s, &s.v_empty[vs], (j / kVStages - 1) & 1)) break;
                mbar_arrive_expect_tx(&s.v_full[vs], 2 * kTileN * 128);
                tc::tma_load_3d(s.v[vs][0], &map_v, 0, j * kTileN, kvh, &s.v_full[vs]);
                tc::tma_load_3d(s.v[vs][1], &map_v, 64, j * kTileN, kvh, &s.v_full[vs]);
                issued = j + 1;
            }
            if (*reinterpret_cast<volatile int *>(&s.abort))
                for (int j = issued > kVStages ? issued - kVStages : 0; j < issued; ++j)
                    mbar_wait(&s.v_full[j % kVStages], (j / kVStages) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_s = tc::idesc_f16(kTileM, kTileN, false, false);
            constexpr uint32_t id_pv = tc::idesc_f16(kTileM, kD, false, true);
            auto s_desc = [&](int ks, int kk, uint64_t &ad, uint64_t &bd) {
                ad = tc::sdesc_sw128(smem_addr(s.q[kk >> 2]) + (kk & 3) * 32, 16, 1024);
                bd = tc::sdesc_sw128(smem_addr(s.k[ks][kk >> 2]) + (kk & 3) * 32, 16, 1024);
            };
            auto issue_s = [&](int j) {   // S_j alone (the first two blocks)
                const int st = j & 1, ks = j % kKStages;
                if (!fa_wait(s, &s.k_full[ks], (j / kKStages) & 1)) return false;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint64_t ad, bd;
                    s_desc(ks, kk, ad, bd);
                    tc::mma_ss(tmem + kColS + st * kTileN, ad, bd, id_s, kk > 0);
                }
                tc::commit(&s.s_full[st]);
                tc::commit(&s.k_empty[ks]);
                return true;
            };
            bool ok = fa_wait(s, &s.q_full, 0) && issue_s(0) && (nkb < 2 || issue_s(1));
            // P_j V_j and S_{j+2} (same S / P / K / V slot st) go out interleaved:
            // two independent accumulator chains keep the tensor pipe busy.
            // The commit after the pair therefore also tells the softmax of
            // block j+2 that P_j V_j is complete.
            for (int j = 0; ok && j < nkb; ++j) {
                const int st = j & 1, vs = j % kVStages, ks = (j + 2) % kKStages;
                const bool s_next = j + 2 < nkb;
                if (!fa_wait(s, &s.p_full[st], (j >> 1) & 1)) break;
                if (!fa_wait(s, &s.v_full[vs], (j / kVStages) & 1)) break;
                if (s_next && !fa_wait(s, &s.k_full[ks], ((j + 2) / kKStages) & 1)) break;
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t vd = tc::sdesc_sw128(smem_addr(s.v[vs][0]) + kk * 2048, 2 * kTileN * 64, 1024);
                    tc::mma_ts(tmem + kColO, tmem + kColP + st * 64 + kk * 8, vd, id_pv, (j > 0) || (kk > 0));
                    if (s_next) {
                        uint64_t ad, bd;
                        s_desc(ks, kk, ad, bd);
                        tc::mma_ss(tmem + kColS + st * kTileN, ad, bd, id_s, kk > 0);
                    }
                }
                tc::commit(&s.o_done[st]);
                tc::commit(&s.v_empty[vs]);
                if (s_next) {
                    tc::commit(&s.s_full[st]);
                    tc::commit(&s.k_empty[ks]);
                }
            }
            // every MMA this thread issued has finished with shared and tensor memory
            // before the CTA frees them (on the abort path too)
            tc::commit(&s.drain);
            mbar_wait(&s.drain, 0);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps
        const int r = 32 * (warp & 3) + lane;   // row within the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const float sc = a.scale_log2;
        float m_ref = -INFINITY;
        // l: sum of the fp32 probabilities (for the log-sum-exp); lr: sum of
        // their fp16 roundings, the weights P V actually applied (normalises O,
        // so each output row is a convex combination of value rows)
        unsigned long long l2a = 0ull, l2b = 0ull, lr2a = 0ull, lr2b = 0ull;
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            const int st = j & 1;
            ok = __all_sync(0xffffffffu, fa_wait(s, &s.s_full[st], (j >> 1) & 1));
            if (!ok) break;
            tc::fence_after_sync();
            uint32_t x[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tc::tmem_ld32(tmem + lane_off + kColS + st * kTileN + 32 * c,
                              *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c]));
            tc::wait_ld();
            if (j == qt) {   // diagonal block: key c > row r is in the future
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c > r) x[c] = __float_as_uint(-INFINITY);
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
                mx0 = fmax3(mx0, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
                mx1 = fmax3(mx1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
                mx2 = fmax3(mx2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
                mx3 = fmax3(mx3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
            }
            const float mxs = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sc;
            float alpha = 1.f;
            const bool grow = mxs > m_ref + kLazyMax;
            if (grow) {
                alpha = ex2(m_ref - mxs);
                m_ref = mxs;
                const unsigned long long al2 = f2pack(alpha, alpha);
                l2a = fmul2(l2a, al2);
                l2b = fmul2(l2b, al2);
                lr2a = fmul2(lr2a, al2);
                lr2b = fmul2(lr2b, al2);
            }
            const unsigned long long sc2 = f2pack(sc, sc), nm2 = f2pack(-m_ref, -m_ref);
            uint32_t p[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                float e0, e1;
                f2unpack(ffma2(f2pack(__uint_as_float(x[2 * c]), __uint_as_float(x[2 * c + 1])), sc2, nm2), e0, e1);
                const float p0 = ex2(e0), p1 = ex2(e1);
                p[c] = pack_half2(p0, p1);
                const float2 pr = unpack_half2(p[c]);
                if (c & 1) {
                    l2b = fadd2(l2b, f2pack(p0, p1));
                    lr2b = fadd2(lr2b, f2pack(pr.x, pr.y));
                } else {
                    l2a = fadd2(l2a, f2pack(p0, p1));
                    lr2a = fadd2(lr2a, f2pack(pr.x, pr.y));
                }
            }
            tc::tmem_st32(tmem + lane_off + kColP + st * 64, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
            tc::tmem_st32(tmem + lane_off + kColP + st * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
            tc::wait_st();
            // O of this warp's rows *= alpha, once P_{j-1} V_{j-1} has landed in O.
            // (P_j over P_{j-2} needs no wait: S_j's commit covered P_{j-2} V_{j-2}.)
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
                ok = __all_sync(0xffffffffu, fa_wait(s, &s.o_done[(j - 1) & 1], ((j - 1) >> 1) & 1));
                if (!ok) break;
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::tmem_ld32(tmem + lane_off + kColO + 32 * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tc::tmem_st32(tmem + lane_off + kColO + 32 * c, o);
                }
                tc::wait_st();
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&s.p_full[st]);
        }
        // ---------------- epilogue: O / l -> fp16 -> swizzled smem (the Q tile) -> TMA store
        if (ok) ok = __all_sync(0xffffffffu, fa_wait(s, &s.o_done[(nkb - 1) & 1], ((nkb - 1) >> 1) & 1));
        if (ok) {
            tc::fence_after_sync();
            float la, lb, ra, rb;
            f2unpack(fadd2(l2a, l2b), la, lb);
            f2unpack(fadd2(lr2a, lr2b), ra, rb);
            const float l = la + lb;
            const float inv = 1.f / (ra + rb);
            const int row = qt * kTileM + r;
            if (row < a.T && row >= a.T - a.W) a.lse2[(size_t)bh * a.W + (row - (a.T - a.W))] = m_ref + log2f(l);
            unsigned char *qbytes = reinterpret_cast<unsigned char *>(s.q);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tc::tmem_ld32(tmem + lane_off + kColO + 32 * c, o);
                tc::wait_ld();
#pragma unroll
                for (int u = 0; u < 4; ++u) {   // 16-byte chunk: d = 32c + 8u .. +7
                    const int d = 32 * c + 8 * u;
                    const int kb = d >> 6, ch = (d & 63) >> 3;
                    uint4 w;
                    w.x = pack_half2(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
                    w.y = pack_half2(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
                    w.z = pack_half2(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
                    w.w = pack_half2(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
                    *reinterpret_cast<uint4 *>(qbytes + kb * (kTileM * 128) + r * 128 + ((ch ^ (r & 7)) << 4)) = w;
                }
            }
            tc::fence_proxy_async_smem();
        }
        asm volatile("bar.sync 1, 128;\n" ::: "memory");
        if (ok && warp == 3 && lane == 0) {
            tc::tma_store_3d(&map_o, s.q[0], 0, qt * kTileM, bh);
            tc::tma_store_3d(&map_o, s.q[1], 64, qt * kTileM, bh);
            tc::bulk_commit_group();
            tc::bulk_wait_all();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
    if (tid == 0 && s.abort) atomicOr(a.status, 1u);
}

// ---------------------------------------------------------------- kernel 2

struct ScoreArgs {
    const uint16_t *q, *k;
    const float *lse2;
    float *scores;
    int Hq, Hkv, T, W;
    float scale_log2;
};

__global__ void __launch_bounds__(128) window_score_kernel(const ScoreArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int gq = a.Hq / a.Hkv;
    const int nrows = gq * a.W;                       // window rows of this KV head
    const int nrows8 = (nrows + 7) / 8 * 8;
    uint16_t *sK = reinterpret_cast<uint16_t *>(smem_raw);   // [64][128]
    uint16_t *sQ = sK + kBN * kD;                              // [nrows8][128]
    float *sL = reinterpret_cast<float *>(sQ + (size_t)nrows8 * kD);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int unit = blockIdx.y;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int j0 = blockIdx.x * kBN;
    const uint16_t *kg = a.k + (size_t)unit * a.T * kD;

    load_tile(sK, kg, j0, kBN, a.T);
    // window rows: row = hh * W + w  <->  q[b, kvh*gq + hh, T - W + w]
    for (int e = tid; e < nrows8 * 16; e += 128) {
        const int r = e >> 4, ch = e & 15;
        const bool ok = r < nrows;
        const int hh = ok ? r / a.W : 0, w = ok ? r % a.W : 0;
        const uint16_t *src = a.q + (((size_t)b * a.Hq + kvh * gq + hh) * a.T + (a.T - a.W + w)) * kD + ch * 8;
        cp_async16(smem_addr(sQ + swz(r, ch * 8)), src, ok);
    }
    cp_async_commit();
    for (int r = tid; r < nrows8; r += 128) {
        if (r < nrows) {
            const int hh = r / a.W, w = r % a.W;
            sL[r] = a.lse2[((size_t)b * a.Hq + kvh * gq + hh) * a.W + w];
        } else {
            sL[r] = INFINITY;   // padding rows contribute exp2(-inf) = 0
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // A = 16 keys of this warp
    uint32_t kf[8][4];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const int r = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int c = 16 * kk + 8 * (lane >> 4);
        ldmatrix_x4(kf[kk], smem_addr(sK + swz(r, c)));
    }
    const int key_a = j0 + 16 * warp + g, key_b = key_a + 8;
    float col_a = 0.f, col_b = 0.f;
    for (int n0 = 0; n0 < nrows8; n0 += 16) {
        const bool two = n0 + 8 < nrows8;
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t bf[4];
            const int rr = n0 + (lane & 7) + (two ? 8 * (lane >> 4) : 0);
            const int c = 16 * kk + 8 * ((lane >> 3) & 1);
            ldmatrix_x4(bf, smem_addr(sQ + swz(rr, c)));
            mma16816(s0, kf[kk], bf[0], bf[1]);
            if (two) mma16816(s1, kf[kk], bf[2], bf[3]);
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            if (half == 1 && !two) break;
            const float *sv = half ? s1 : s0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = n0 + 8 * half + 2 * t + (i & 1);
                const int key = (i >> 1) ? key_b : key_a;
                const int qpos = a.T - a.W + (row % a.W);
                float p = 0.f;
                if (row < nrows && key <= qpos) p = exp2f(sv[i] * a.scale_log2 - sL[row]);
                if (i >> 1) col_b += p;
                else col_a += p;
            }
        }
    }
    col_a += __shfl_xor_sync(0xffffffffu, col_a, 1);
    col_a += __shfl_xor_sync(0xffffffffu, col_a, 2);
    col_b += __shfl_xor_sync(0xffffffffu, col_b, 1);
    col_b += __shfl_xor_sync(0xffffffffu, col_b, 2);
    if (t == 0) {
        float *sc = a.scores + (size_t)unit * a.T;
        if (key_a < a.T) sc[key_a] = col_a;
        if (key_b < a.T) sc[key_b] = col_b;
    }
}

// Shared-memory opt-ins, per device (a function attribute applies to the device
// current when it is set), guarded for calls from several host threads.
std::mutex g_attr_mu;
bool g_attr_fa[kMaxDevices] = {};
size_t g_attr_score[kMaxDevices] = {};

std::mutex g_encode_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// [planes][rows][128] fp16, 128-byte swizzled boxes of 64 x 128 rows
int make_map(CUtensorMap *m, const void *base, int rows, int planes, const char *what) {
    {
        std::lock_guard<std::mutex> lk(g_encode_mu);
        if (!g_encode) {
            cudaDriverEntryPointQueryResult qr;
            void *fn = nullptr;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
                qr != cudaDriverEntryPointSuccess || !fn)
                return fail(MINIKV_ERR_CUDA, "select_prefill: cuTensorMapEncodeTiled unavailable");
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)rows, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)rows * kD * 2};
    cuuint32_t box[3] = {64, 128, 1}, estr[3] = {1, 1, 1};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MINIKV_ERR_CUDA, "select_prefill: tensor map for %s (CUresult %d)", what, (int)r);
    return 0;
}

}  // namespace

// Workspace: the window rows' log-sum-exp [B, Hq, W] fp32, then a 256-byte
// block whose first word is the call's status (see minikv_select_prefill_status).
size_t prefill_lse_bytes(int B, int Hq, int W) { return ((size_t)B * Hq * W * 4 + 255) / 256 * 256; }
size_t prefill_workspace_bytes(int B, int Hq, int W) { return prefill_lse_bytes(B, Hq, W) + 256; }

int prefill_launch(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int Hq, int Hkv, int T, int W,
                   float sm_scale, uint16_t *o, float *scores, void *ws, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mo;
    int rc;
    if ((rc = make_map(&mq, q, T, B * Hq, "q")) || (rc = make_map(&mk, k, T, B * Hkv, "k")) ||
        (rc = make_map(&mv, v, T, B * Hkv, "v")) || (rc = make_map(&mo, o, T, B * Hq, "o")))
        return rc;
    FaArgs fa;
    fa.lse2 = static_cast<float *>(ws);
    fa.status = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + prefill_lse_bytes(B, Hq, W));
    if (cudaMemsetAsync(fa.status, 0, sizeof(unsigned), stream) != cudaSuccess)
        return check_launch("select_prefill: clearing the status word");
    fa.Hq = Hq; fa.Hkv = Hkv; fa.T = T; fa.W = W;
    fa.nqt = (T + kTileM - 1) / kTileM;
    {   // K and V of one (sequence, head): 2 x T x 128 fp16; about 64 MB of them per group
        const long long per = 512ll * T;
        long long hg = (64ll << 20) / per;
        if (hg < 1) hg = 1;
        if (hg > (long long)B * Hq) hg = (long long)B * Hq;
        fa.hg = (int)hg;
    }
    fa.scale_log2 = sm_scale * kLog2e;
    const size_t fa_smem = sizeof(FaSmem) + 1024;
    const int dev = current_device();
    if (dev < 0) return check_launch("select_prefill: cudaGetDevice");
    {
        std::lock_guard<std::mutex> lk(g_attr_mu);
        if (!g_attr_fa[dev]) {
            if (cudaFuncSetAttribute(fa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fa_smem) !=
                cudaSuccess)
                return check_launch("select_prefill: attribute");
            g_attr_fa[dev] = true;
        }
    }
    fa_tc_kernel<<<(unsigned)(fa.nqt * B * Hq), kFaThreads, fa_smem, stream>>>(mq, mk, mv, mo, fa);
    rc = check_launch("select_prefill: flash attention");
    if (rc) return rc;

    ScoreArgs sa;
    sa.q = q; sa.k = k; sa.lse2 = fa.lse2; sa.scores = scores;
    sa.Hq = Hq; sa.Hkv = Hkv; sa.T = T; sa.W = W;
    sa.scale_log2 = fa.scale_log2;
    const int nrows8 = ((Hq / Hkv) * W + 7) / 8 * 8;
    const size_t sc_smem = (size_t)kBN * kD * 2 + (size_t)nrows8 * kD * 2 + (size_t)nrows8 * 4;
    {
        std::lock_guard<std::mutex> lk(g_attr_mu);
        if (sc_smem > g_attr_score[dev]) {
            if (cudaFuncSetAttribute(window_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)sc_smem) != cudaSuccess)
                return check_launch("select_prefill: attribute");
            g_attr_score[dev] = sc_smem;
        }
    }
    window_score_kernel<<<dim3((T + kBN - 1) / kBN, B * Hkv), 128, sc_smem, stream>>>(sa);
    return check_launch("select_prefill: window scores");
}

}  // namespace minikv
