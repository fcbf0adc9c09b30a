// minikv_decode_attn: one decoding step over the 2-bit cache (flash-decoding).
//
// Source: MiniKV abstract (specialized CUDA kernels compatible with
// FlashAttention) and the gptget.net summary of arXiv 2411.18077, section
// 方法论 (sub-channel key / per-token value 2-bit quantization, compact layout).
//
// One launch per layer-step.  CTA (x = 0, unit) attends over the fp16 residual
// (and appends the new token, and flushes a full key group); CTAs (x >= 1,
// unit) each attend over one contiguous chunk of packed tokens.  Each CTA
// writes its partial softmax state (m, l, sum p*v) to the workspace; the last
// CTA of a unit (atomic arrival counter, self-resetting) merges them.
//
// Packed chunk, per warp and 32-token slice (one key group), heads of one KV
// head taken four at a time (g <= 4):
//   scores  S[token, col] = sum_c a[token, c] * b[c, col]          (mma m16n8k16)
//     a = 1 + code * 2^(p-10): the 2-bit code dropped into an fp16 mantissa at
//         bit p (6 or 8) by one AND/OR -- no integer->float conversion;
//     b = q * k_scale * 2^(10-p), split hi + lo in fp16: cols 0..3 carry the hi
//         parts of heads 0..3, cols 4..7 the lo parts, so one mma gives a
//         22-bit-accurate product for four heads;
//     score_h = S[., h] + S[., h+4] - sum_c b_c + sum_c q_c * k_zero_c.
//   output  O^T[channel, col] = sum_t a'[channel, t] * P'[t, col]    (mma)
//     a' = the value code in the same mantissa form; P' = p_t * v_scale_t split
//     hi/lo the same way, moved from the score fragment layout into the B
//     operand layout with movmatrix; out = (O^T - sum P') * 2^(10-p) + sum p*v_zero.
// The token order inside a 16-token m-tile is permuted (kPerm) so that both
// the key-word loads and the value-word loads of a warp hit 32 distinct banks.
#include <math.h>

#include "common.cuh"

namespace minikv {

namespace {

constexpr int kTile = 128;   // packed tokens per shared-memory stage (4 warps x 32)
constexpr int kStages = 3;
constexpr int kThreads = 128;
constexpr int kPartStride = 132;   // floats per (unit, split, head): y[128], m, l

struct __align__(16) Tile {
    uint32_t kc[kTile * 8];
    uint32_t vc[kTile * 8];
    uint16_t ks[4 * kD];
    uint16_t kz[4 * kD];
    uint16_t vs[kTile];
    uint16_t vz[kTile];
};

struct __align__(16) Smem {
    Tile tile[kStages];
    uint64_t full[kStages];
    float wm[4][4], wl[4][4];
    float wy[4][4][kD];
    int flag;
};

struct Args {
    const uint32_t *k_codes, *v_codes;
    const uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
    uint32_t *k_codes_w, *v_codes_w;
    uint16_t *k_scale_w, *k_zero_w, *v_scale_w, *v_zero_w;
    uint16_t *k_res, *v_res;
    const uint16_t *q, *k_new, *v_new;
    uint16_t *out;
    float *part;
    unsigned *counters;
    int *err;
    int Hkv, g, G, cap, ring;
    int n_q, r, res_start, flush;
    int chunk, S;
    float scale_log2;
};

// row permutation inside an 8-row half of an m-tile (see file comment)
__device__ __forceinline__ int perm8(int r) {
    return (0x57461320u >> (4 * r)) & 0xf;   // {0,2,1,3,6,4,7,5}
}

template <int S>
__device__ __forceinline__ uint32_t shiftr(uint32_t x) {
    if constexpr (S >= 0) return x >> S;
    else return x << (-S);
}

__device__ __forceinline__ uint32_t magic(uint32_t x, uint32_t mask) {
    return (x & mask) | 0x3C003C00u;   // fp16 1.0 in both halves + the code bits
}

__device__ __forceinline__ float warp_sum_g(float x) {   // over lanes with equal t (xor 4, 8, 16)
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    x += __shfl_xor_sync(0xffffffffu, x, 8);
    x += __shfl_xor_sync(0xffffffffu, x, 16);
    return x;
}
__device__ __forceinline__ float warp_max_g(float x) {
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
    x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
    return x;
}

// Write this CTA's partial state for `unit`, split `split`, then let the last
// arriving CTA of the unit merge all splits into `out`.
__device__ void finish_unit(const Args &a, Smem &sm, int unit, int split, const float *m_h, const float *l_h,
                            const float (*y_h)[kD]) {
    const int tid = threadIdx.x;
    float *base = a.part + ((size_t)unit * a.S + split) * 4 * kPartStride;
    for (int h = 0; h < a.g; ++h) {
        base[h * kPartStride + tid] = y_h[h][tid];
        if (tid == 0) {
            base[h * kPartStride + 128] = m_h[h];
            base[h * kPartStride + 129] = l_h[h];
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.flag = (atomicInc(&a.counters[unit], (unsigned)(a.S - 1)) == (unsigned)(a.S - 1));
    __syncthreads();
    if (!sm.flag) return;
    __threadfence();
    const float *ub = a.part + (size_t)unit * a.S * 4 * kPartStride;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int Hq = a.Hkv * a.g;
    for (int h = 0; h < a.g; ++h) {
        float M = -INFINITY;
        for (int s = 0; s < a.S; ++s) M = fmaxf(M, __ldcg(ub + (s * 4 + h) * kPartStride + 128));
        float L = 0.f, Y = 0.f;
        for (int s = 0; s < a.S; ++s) {
            const float *p = ub + (s * 4 + h) * kPartStride;
            float ms = __ldcg(p + 128);
            float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
            L += f * __ldcg(p + 129);
            Y += f * __ldcg(p + tid);
        }
        a.out[((size_t)b * Hq + kvh * a.g + h) * kD + tid] = f2h(Y / L);
    }
}

// ---------------------------------------------------------------- residual CTA

__device__ void residual_cta(const Args &a, Smem &sm, int unit) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int Hq = a.Hkv * a.g;
    const uint16_t *knew = a.k_new + (size_t)unit * kD;
    const uint16_t *vnew = a.v_new + (size_t)unit * kD;
    uint16_t *kres = a.k_res + (size_t)unit * a.ring * kD;
    uint16_t *vres = a.v_res + (size_t)unit * a.ring * kD;
    const int r = a.r;
    auto slot = [&](int i) { int s = a.res_start + i; return s >= a.ring ? s - a.ring : s; };
    auto krow = [&](int i) -> const uint16_t * { return i == r - 1 ? knew : kres + (size_t)slot(i) * kD; };
    auto vrow = [&](int i) -> const uint16_t * { return i == r - 1 ? vnew : vres + (size_t)slot(i) * kD; };

    // append: the new token goes to ring slot of logical index r-1
    if (tid < 16) {
        reinterpret_cast<uint4 *>(kres + (size_t)slot(r - 1) * kD)[tid] = reinterpret_cast<const uint4 *>(knew)[tid];
    } else if (tid < 32) {
        reinterpret_cast<uint4 *>(vres + (size_t)slot(r - 1) * kD)[tid - 16] =
            reinterpret_cast<const uint4 *>(vnew)[tid - 16];
    }

    // shared scratch (the stage buffers are unused by this CTA)
    float *qs = reinterpret_cast<float *>(&sm.tile[0]);     // [4][128]
    float *sc = qs + 4 * kD;                                  // [4][ring]
    for (int i = tid; i < a.g * kD; i += kThreads) {
        int h = i / kD, c = i % kD;
        qs[i] = h2f(a.q[((size_t)b * Hq + kvh * a.g + h) * kD + c]);
    }
    __syncthreads();
    // scores: warp per token, lane per 4 channels
    for (int i = warp; i < r; i += 4) {
        uint2 raw = *reinterpret_cast<const uint2 *>(krow(i) + 4 * lane);
        float k0 = h2f(raw.x & 0xffff), k1 = h2f(raw.x >> 16), k2 = h2f(raw.y & 0xffff), k3 = h2f(raw.y >> 16);
        for (int h = 0; h < a.g; ++h) {
            const float *qh = qs + h * kD + 4 * lane;
            float d = qh[0] * k0 + qh[1] * k1 + qh[2] * k2 + qh[3] * k3;
            for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            if (lane == 0) sc[h * a.ring + i] = d * a.scale_log2;
        }
    }
    __syncthreads();
    // softmax per head (warp h)
    if (warp < a.g) {
        float *s = sc + warp * a.ring;
        float m = -INFINITY;
        for (int i = lane; i < r; i += 32) m = fmaxf(m, s[i]);
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int i = lane; i < r; i += 32) {
            float p = exp2f(s[i] - m);
            s[i] = p;
            l += p;
        }
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (lane == 0) {
            sm.wm[0][warp] = m;
            sm.wl[0][warp] = l;
        }
    }
    __syncthreads();
    // values: thread per channel
    for (int h = 0; h < a.g; ++h) sm.wy[0][h][tid] = 0.f;
    {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i < r; ++i) {
            float v = h2f(vrow(i)[tid]);
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (h < a.g) acc[h] += sc[h * a.ring + i] * v;
        }
        for (int h = 0; h < a.g; ++h) sm.wy[0][h][tid] = acc[h];
    }
    __syncthreads();

    if (a.flush) {
        // the oldest G residual tokens become key group n_q/G and G value tokens
        const size_t tok0 = (size_t)unit * a.cap + a.n_q;
        pack_key_group(krow, a.G, a.k_codes_w + tok0 * 8,
                       a.k_scale_w + ((size_t)unit * (a.cap / a.G) + a.n_q / a.G) * kD,
                       a.k_zero_w + ((size_t)unit * (a.cap / a.G) + a.n_q / a.G) * kD);
        pack_value_tokens(vrow, a.G, kD, a.v_codes_w + tok0 * 8, a.v_scale_w + tok0, a.v_zero_w + tok0);
    }
    finish_unit(a, sm, unit, 0, sm.wm[0], sm.wl[0], sm.wy[0]);
}

// ------------------------------------------------------------------ packed CTA

__device__ void issue_tile(const Args &a, Smem &sm, int stage, int unit, int t0, int n) {
    Tile &T = sm.tile[stage];
    const size_t tok = (size_t)unit * a.cap + t0;
    const int gfirst = t0 / a.G, glast = (t0 + n - 1) / a.G;
    const int ng = glast - gfirst + 1;
    const uint32_t bytes = n * 32u * 2u + ng * kD * 2u * 2u + n * 2u * 2u;
    mbar_arrive_expect_tx(&sm.full[stage], bytes);
    bulk_g2s(T.kc, a.k_codes + tok * 8, n * 32u, &sm.full[stage]);
    bulk_g2s(T.vc, a.v_codes + tok * 8, n * 32u, &sm.full[stage]);
    const size_t grow = (size_t)unit * (a.cap / a.G) + gfirst;
    bulk_g2s(T.ks, a.k_scale + grow * kD, ng * kD * 2u, &sm.full[stage]);
    bulk_g2s(T.kz, a.k_zero + grow * kD, ng * kD * 2u, &sm.full[stage]);
    bulk_g2s(T.vs, a.v_scale + tok, n * 2u, &sm.full[stage]);
    bulk_g2s(T.vz, a.v_zero + tok, n * 2u, &sm.full[stage]);
}

__device__ void packed_cta(const Args &a, Smem &sm, int unit, int chunk_idx) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g_ = lane >> 2, t_ = lane & 3;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int Hq = a.Hkv * a.g;
    const int c0 = chunk_idx * a.chunk;
    const int c1 = min(c0 + a.chunk, a.n_q);
    const int ntiles = (c1 - c0 + kTile - 1) / kTile;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0)
        for (int s = 0; s < kStages && s < ntiles; ++s) issue_tile(a, sm, s, unit, c0 + s * kTile, min(kTile, c1 - c0 - s * kTile));

    // q * 2^(10-p) for the B-operand channels of this lane (head g_ & 3)
    const int hq = g_ & 3;
    const bool lo_col = g_ >= 4;
    float qw[8][4];
    {
        const bool live = hq < a.g;
        const uint16_t *qp = a.q + ((size_t)b * Hq + kvh * a.g + (live ? hq : 0)) * kD;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c00 = 16 * (2 * t_ + (kk >> 2)) + 2 * (kk & 3);
            qw[kk][0] = live ? h2f(qp[c00]) * 16.f : 0.f;
            qw[kk][1] = live ? h2f(qp[c00 + 8]) * 16.f : 0.f;
            qw[kk][2] = live ? h2f(qp[c00 + 1]) * 4.f : 0.f;
            qw[kk][3] = live ? h2f(qp[c00 + 9]) * 4.f : 0.f;
        }
    }
    // running state: heads hA = 2*(t_&1) + e, e = 0, 1
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, pz[2] = {0.f, 0.f}, ps[2] = {0.f, 0.f};
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    const int hA = 2 * (t_ & 1);
    const int pg = perm8(g_);
    const int p2t = perm8(2 * t_), p2t1 = perm8(2 * t_ + 1);

    for (int it = 0; it < ntiles; ++it) {
        const int stage = it % kStages;
        const int t0 = c0 + it * kTile;
        const int n = min(kTile, c1 - t0);
        bool ok = mbar_wait(&sm.full[stage], (it / kStages) & 1);
        Tile &T = sm.tile[stage];
        if (ok && 32 * warp < n) {
            // ---- key group setup: B fragments and the per-head constant
            const int grp = (t0 + 32 * warp) / a.G - t0 / a.G;
            const uint16_t *ksr = T.ks + grp * kD, *kzr = T.kz + grp * kD;
            uint32_t bk[8][2];
            float part_b = 0.f, qz6 = 0.f, qz8 = 0.f;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c00 = 16 * (2 * t_ + (kk >> 2)) + 2 * (kk & 3);
                float x0 = qw[kk][0] * h2f(ksr[c00]), x1 = qw[kk][1] * h2f(ksr[c00 + 8]);
                float x2 = qw[kk][2] * h2f(ksr[c00 + 1]), x3 = qw[kk][3] * h2f(ksr[c00 + 9]);
                uint32_t h01 = pack_half2(x0, x1), h23 = pack_half2(x2, x3);
                if (lo_col) {
                    float2 f01 = unpack_half2(h01), f23 = unpack_half2(h23);
                    h01 = pack_half2(x0 - f01.x, x1 - f01.y);
                    h23 = pack_half2(x2 - f23.x, x3 - f23.y);
                }
                bk[kk][0] = h01;
                bk[kk][1] = h23;
                float2 u = unpack_half2(h01), v = unpack_half2(h23);
                part_b += (u.x + u.y) + (v.x + v.y);
                qz6 += qw[kk][0] * h2f(kzr[c00]) + qw[kk][1] * h2f(kzr[c00 + 8]);
                qz8 += qw[kk][2] * h2f(kzr[c00 + 1]) + qw[kk][3] * h2f(kzr[c00 + 9]);
            }
            float cst = (lo_col ? 0.f : (qz6 * 0.0625f + qz8 * 0.25f)) - part_b;
            cst += __shfl_xor_sync(0xffffffffu, cst, 1);
            cst += __shfl_xor_sync(0xffffffffu, cst, 2);
            cst += __shfl_xor_sync(0xffffffffu, cst, 16);
            const float cA = __shfl_sync(0xffffffffu, cst, 4 * hA);
            const float cB = __shfl_sync(0xffffffffu, cst, 4 * (hA + 1));

            // ---- scores for the two m-tiles
            float x[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int rowg = 32 * warp + 16 * mt + pg;
                const uint2 ka = *reinterpret_cast<const uint2 *>(&T.kc[rowg * 8 + 2 * t_]);
                const uint2 kb = *reinterpret_cast<const uint2 *>(&T.kc[(rowg + 8) * 8 + 2 * t_]);
                float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t wa = (kk < 4) ? ka.x : ka.y, wb = (kk < 4) ? kb.x : kb.y;
                    uint32_t sa, sb;
                    switch (kk & 3) {
                        case 0: sa = shiftr<-6>(wa); sb = shiftr<-6>(wb); break;
                        case 1: sa = shiftr<-2>(wa); sb = shiftr<-2>(wb); break;
                        case 2: sa = shiftr<2>(wa); sb = shiftr<2>(wb); break;
                        default: sa = shiftr<6>(wa); sb = shiftr<6>(wb); break;
                    }
                    uint32_t af[4] = {magic(sa, 0x00C000C0u), magic(sb, 0x00C000C0u), magic(sa, 0x03000300u),
                                      magic(sb, 0x03000300u)};
                    mma16816(s, af, bk[kk][0], bk[kk][1]);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v = s[i] + __shfl_xor_sync(0xffffffffu, s[i], 2);
                    x[mt][i] = (v + ((i & 1) ? cB : cA)) * a.scale_log2;
                }
            }
            // ---- online softmax update (per head e = 0, 1)
            float alpha[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mx = fmaxf(fmaxf(x[0][e], x[0][e + 2]), fmaxf(x[1][e], x[1][e + 2]));
                mx = warp_max_g(mx);
                const float mn = fmaxf(m_run[e], mx);
                alpha[e] = exp2f(m_run[e] - mn);
                m_run[e] = mn;
                l_run[e] *= alpha[e];
                pz[e] *= alpha[e];
                ps[e] *= alpha[e];
            }
#pragma unroll
            for (int nu = 0; nu < 8; ++nu) {
                acc[nu][0] *= alpha[0];
                acc[nu][1] *= alpha[1];
                acc[nu][2] *= alpha[0];
                acc[nu][3] *= alpha[1];
            }
            // ---- P' = p * v_scale (hi on lanes t<2, lo on t>=2), then O^T += V'^T P'
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int base = 32 * warp + 16 * mt;
                uint32_t prow[2];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {   // row g (hr=0) and row g+8 (hr=1)
                    const int tok = base + 8 * hr + pg;
                    const float vsc = h2f(T.vs[tok]), vzr = h2f(T.vz[tok]);
                    const float p0 = exp2f(x[mt][2 * hr] - m_run[0]);
                    const float p1 = exp2f(x[mt][2 * hr + 1] - m_run[1]);
                    l_run[0] += p0;
                    l_run[1] += p1;
                    pz[0] += p0 * vzr;
                    pz[1] += p1 * vzr;
                    const float y0 = p0 * vsc, y1 = p1 * vsc;
                    uint32_t hv = pack_half2(y0, y1);
                    if (t_ >= 2) {
                        float2 f = unpack_half2(hv);
                        hv = pack_half2(y0 - f.x, y1 - f.y);
                    }
                    float2 f = unpack_half2(hv);
                    ps[0] += f.x;
                    ps[1] += f.y;
                    prow[hr] = hv;
                }
                const uint32_t bv0 = movmatrix_t(prow[0]), bv1 = movmatrix_t(prow[1]);
                const uint32_t wA = T.vc[(base + p2t) * 8 + g_], wB = T.vc[(base + p2t1) * 8 + g_];
                const uint32_t wC = T.vc[(base + 8 + p2t) * 8 + g_], wD = T.vc[(base + 8 + p2t1) * 8 + g_];
                const uint32_t lo1 = __byte_perm(wA, wB, 0x5410), hi1 = __byte_perm(wA, wB, 0x7632);
                const uint32_t lo2 = __byte_perm(wC, wD, 0x5410), hi2 = __byte_perm(wC, wD, 0x7632);
#pragma unroll
                for (int pr = 0; pr < 4; ++pr) {
                    uint32_t s1, s2, s3, s4;
                    switch (pr) {
                        case 0: s1 = shiftr<-6>(lo1); s2 = shiftr<-6>(hi1); s3 = shiftr<-6>(lo2); s4 = shiftr<-6>(hi2); break;
                        case 1: s1 = shiftr<-2>(lo1); s2 = shiftr<-2>(hi1); s3 = shiftr<-2>(lo2); s4 = shiftr<-2>(hi2); break;
                        case 2: s1 = shiftr<2>(lo1); s2 = shiftr<2>(hi1); s3 = shiftr<2>(lo2); s4 = shiftr<2>(hi2); break;
                        default: s1 = shiftr<6>(lo1); s2 = shiftr<6>(hi1); s3 = shiftr<6>(lo2); s4 = shiftr<6>(hi2); break;
                    }
                    uint32_t a6[4] = {magic(s1, 0x00C000C0u), magic(s2, 0x00C000C0u), magic(s3, 0x00C000C0u),
                                      magic(s4, 0x00C000C0u)};
                    mma16816(acc[2 * pr], a6, bv0, bv1);
                    uint32_t a8[4] = {magic(s1, 0x03000300u), magic(s2, 0x03000300u), magic(s3, 0x03000300u),
                                      magic(s4, 0x03000300u)};
                    mma16816(acc[2 * pr + 1], a8, bv0, bv1);
                }
            }
        }
        const int timed_out = __syncthreads_or(!ok);
        if (timed_out) {
            if (tid == 0 && a.err) atomicExch(a.err, 1);
            break;
        }
        if (tid == 0 && it + kStages < ntiles)
            issue_tile(a, sm, stage, unit, t0 + kStages * kTile, min(kTile, c1 - t0 - kStages * kTile));
    }

    // ---- warp epilogue: y[channel][head] = (acc - sum P') * 2^(10-p) + sum p*zero
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        l_run[e] = warp_sum_g(l_run[e]);
        pz[e] = warp_sum_g(pz[e]);
        ps[e] = warp_sum_g(ps[e]);
    }
#pragma unroll
    for (int nu = 0; nu < 8; ++nu) {
        const float w = (nu & 1) ? 4.f : 16.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float y = (acc[nu][i] - ps[i & 1]) * w;
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            acc[nu][i] = y + pz[i & 1];
        }
    }
    if (t_ < 2) {
#pragma unroll
        for (int nu = 0; nu < 8; ++nu) {
            const int ch = 16 * g_ + nu;
            sm.wy[warp][hA][ch] = acc[nu][0];
            sm.wy[warp][hA + 1][ch] = acc[nu][1];
            sm.wy[warp][hA][ch + 8] = acc[nu][2];
            sm.wy[warp][hA + 1][ch + 8] = acc[nu][3];
        }
        if (g_ == 0) {
            sm.wm[warp][hA] = m_run[0];
            sm.wm[warp][hA + 1] = m_run[1];
            sm.wl[warp][hA] = l_run[0];
            sm.wl[warp][hA + 1] = l_run[1];
        }
    }
    __syncthreads();
    // ---- merge the 4 warps (thread = channel)
    float mh[4], lh[4];
    for (int h = 0; h < 4; ++h) {
        float M = fmaxf(fmaxf(sm.wm[0][h], sm.wm[1][h]), fmaxf(sm.wm[2][h], sm.wm[3][h]));
        float L = 0.f, Y = 0.f;
        for (int w = 0; w < 4; ++w) {
            float f = (sm.wm[w][h] == -INFINITY) ? 0.f : exp2f(sm.wm[w][h] - M);
            L += f * sm.wl[w][h];
            Y += f * sm.wy[w][h][tid];
        }
        mh[h] = M;
        lh[h] = L;
        __syncthreads();
        sm.wy[0][h][tid] = Y;   // wy[0][h] is only read by this thread for this h
        __syncthreads();
    }
    finish_unit(a, sm, unit, 1 + chunk_idx, mh, lh, sm.wy[0]);
}

__global__ void __launch_bounds__(kThreads) decode_kernel(const Args a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    const int unit = blockIdx.y;
    if (blockIdx.x == 0) residual_cta(a, sm, unit);
    else packed_cta(a, sm, unit, blockIdx.x - 1);
}

int g_num_sms = 0;

}  // namespace

// Number of CTAs the launch splits a unit's packed tokens into.
static void plan_chunks(int units, int n_q, int &n_chunks, int &chunk) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    n_chunks = 0;
    chunk = kTile;
    if (n_q <= 0) return;
    const int target = 2 * 4 * g_num_sms;        // about two waves at 4 CTAs per SM
    int want = target / units - 1;
    if (want < 1) want = 1;
    const int max_chunks = (n_q + kTile - 1) / kTile;
    n_chunks = want < max_chunks ? want : max_chunks;
    chunk = (n_q + n_chunks - 1) / n_chunks;
    chunk = (chunk + 31) / 32 * 32;
    n_chunks = (n_q + chunk - 1) / chunk;
}

size_t decode_workspace_bytes(int B, int Hkv, int max_tokens) {
    const size_t units = (size_t)B * Hkv;
    const size_t S = 1 + (size_t)(max_tokens + kTile - 1) / kTile;
    return ((units * 4 + 255) / 256) * 256 + units * S * 4 * kPartStride * 4;
}

// Bytes of the workspace prefix that holds the per-unit arrival counters.
size_t decode_counter_bytes(int B, int Hkv) { return (((size_t)B * Hkv * 4 + 255) / 256) * 256; }

// Workspace bytes the next decode call on this cache state will use.
size_t decode_call_workspace_bytes(const minikv_cache *c) {
    const int units = c->B * c->Hkv;
    int n_chunks, chunk;
    plan_chunks(units, c->n_packed, n_chunks, chunk);
    return decode_counter_bytes(c->B, c->Hkv) + (size_t)units * (1 + n_chunks) * 4 * kPartStride * 4;
}

int decode_launch(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                  float sm_scale, uint16_t *out, void *ws, size_t ws_bytes, cudaStream_t stream) {
    const int units = c->B * c->Hkv;
    const int g = Hq / c->Hkv;
    const int ring = c->R + c->G;
    const int r = c->n_res + 1;
    const int flush = (r == ring) ? 1 : 0;
    if (flush && c->n_packed + c->G > c->cap)
        return fail(MINIKV_ERR_CAPACITY, "decode_attn: flushing a key group would exceed cap=%d", c->cap);
    int n_chunks, chunk;
    plan_chunks(units, c->n_packed, n_chunks, chunk);
    const int S = 1 + n_chunks;
    const size_t cnt_bytes = (((size_t)units * 4 + 255) / 256) * 256;
    const size_t need = cnt_bytes + (size_t)units * S * 4 * kPartStride * 4;
    if (ws == nullptr || ws_bytes < need)
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: workspace of %zu bytes needed, %zu given", need, ws_bytes);

    Args a;
    a.k_codes = c->k_codes; a.v_codes = c->v_codes;
    a.k_scale = c->k_scale; a.k_zero = c->k_zero; a.v_scale = c->v_scale; a.v_zero = c->v_zero;
    a.k_codes_w = c->k_codes; a.v_codes_w = c->v_codes;
    a.k_scale_w = c->k_scale; a.k_zero_w = c->k_zero; a.v_scale_w = c->v_scale; a.v_zero_w = c->v_zero;
    a.k_res = c->k_res; a.v_res = c->v_res;
    a.q = q; a.k_new = k_new; a.v_new = v_new; a.out = out;
    a.counters = reinterpret_cast<unsigned *>(ws);
    a.part = reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes);
    a.err = nullptr;
    a.Hkv = c->Hkv; a.g = g; a.G = c->G; a.cap = c->cap; a.ring = ring;
    a.n_q = c->n_packed; a.r = r; a.res_start = c->res_start; a.flush = flush;
    a.chunk = chunk; a.S = S;
    a.scale_log2 = sm_scale * kLog2e;

    const size_t smem = sizeof(Smem);
    static bool attr_done = false;
    if (!attr_done) {
        if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return check_launch("decode_attn: cudaFuncSetAttribute");
        attr_done = true;
    }
    dim3 grid(S, units);
    decode_kernel<<<grid, kThreads, smem, stream>>>(a);
    int rc = check_launch("decode_attn");
    if (rc) return rc;
    // host-side state
    c->n_res = r;
    if (flush) {
        c->n_packed += c->G;
        c->n_res -= c->G;
        c->res_start = (c->res_start + c->G) % ring;
    }
    return MINIKV_OK;
}

}  // namespace minikv
