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
// Kernel 1 (fa_fwd_kernel): 64 query rows x 64 keys per step, 4 warps of 16
// rows, fp16 mma.sync with fp32 accumulation, K/V double-buffered by cp.async
// in XOR-swizzled shared memory.  Kernel 2 (window_score_kernel): one CTA per
// 64 keys of one KV head; S^T = K Q_w^T on the tensor cores, then column sums.
#include <math.h>

#include "common.cuh"

namespace minikv {

namespace {

constexpr int kBM = 64, kBN = 64;

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

struct FaArgs {
    const uint16_t *q, *k, *v;
    uint16_t *o;
    float *lse2;   // [B, Hq, W] window rows, log2 domain
    int Hq, Hkv, T, W;
    float scale_log2;
};

__global__ void __launch_bounds__(128) fa_fwd_kernel(const FaArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint16_t *sQ = reinterpret_cast<uint16_t *>(smem_raw);
    uint16_t *sK = sQ + kBM * kD;          // [2][64][128]
    uint16_t *sV = sK + 2 * kBN * kD;      // [2][64][128]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int nqt = (a.T + kBM - 1) / kBM;
    const int qt = nqt - 1 - blockIdx.x;    // heaviest tiles first
    const int bh = blockIdx.y;
    const int b = bh / a.Hq, h = bh % a.Hq;
    const int kvh = h / (a.Hq / a.Hkv);
    const uint16_t *qg = a.q + (size_t)bh * a.T * kD;
    const uint16_t *kg = a.k + ((size_t)b * a.Hkv + kvh) * a.T * kD;
    const uint16_t *vg = a.v + ((size_t)b * a.Hkv + kvh) * a.T * kD;
    const int q0 = qt * kBM;
    const int nkb = qt + 1;   // causal: key blocks 0..qt

    load_tile(sQ, qg, q0, kBM, a.T);
    cp_async_commit();
    load_tile(sK, kg, 0, kBN, a.T);
    load_tile(sV, vg, 0, kBN, a.T);
    cp_async_commit();

    uint32_t qf[8][4];
    float oacc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, lr[2] = {0.f, 0.f};
    const int row_g = q0 + 16 * warp + g;   // this lane's rows: row_g and row_g + 8

    for (int kb = 0; kb < nkb; ++kb) {
        cp_async_wait<0>();
        __syncthreads();
        if (kb + 1 < nkb) {
            load_tile(sK + ((kb + 1) & 1) * kBN * kD, kg, (kb + 1) * kBN, kBN, a.T);
            load_tile(sV + ((kb + 1) & 1) * kBN * kD, vg, (kb + 1) * kBN, kBN, a.T);
            cp_async_commit();
        }
        if (kb == 0) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int r = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int c = 16 * kk + 8 * (lane >> 4);
                ldmatrix_x4(qf[kk], smem_addr(sQ + swz(r, c)));
            }
        }
        const uint16_t *Kb = sK + (kb & 1) * kBN * kD;
        const uint16_t *Vb = sV + (kb & 1) * kBN * kD;
        // S = Q K^T: 16 rows x 64 keys per warp
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {   // pairs of 8-key n-tiles
                uint32_t bf[4];
                const int r = 16 * np + (lane & 7) + 8 * (lane >> 4);
                const int c = 16 * kk + 8 * ((lane >> 3) & 1);
                ldmatrix_x4(bf, smem_addr(Kb + swz(r, c)));
                mma16816(s[2 * np], qf[kk], bf[0], bf[1]);
                mma16816(s[2 * np + 1], qf[kk], bf[2], bf[3]);
            }
        }
        // online softmax (log2 domain), causal mask on the diagonal block
        const bool diag = (kb == qt);
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float x = s[nt][i] * a.scale_log2;
                if (diag) {
                    const int key = kb * kBN + 8 * nt + 2 * t + (i & 1);
                    const int row = row_g + 8 * (i >> 1);
                    if (key > row) x = -INFINITY;
                }
                s[nt][i] = x;
                mx[i >> 1] = fmaxf(mx[i >> 1], x);
            }
        float alpha[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
            const float mn = fmaxf(m[e], mx[e]);
            alpha[e] = exp2f(m[e] - mn);
            m[e] = mn;
            l[e] *= alpha[e];
            lr[e] *= alpha[e];
        }
        uint32_t pf[4][4];   // P as the A operand of P V: 4 k-chunks of 16 keys
        float ls[2] = {0.f, 0.f}, lrs[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float p0 = exp2f(s[nt][0] - m[0]), p1 = exp2f(s[nt][1] - m[0]);
            const float p2 = exp2f(s[nt][2] - m[1]), p3 = exp2f(s[nt][3] - m[1]);
            const uint32_t h01 = pack_half2(p0, p1), h23 = pack_half2(p2, p3);
            const float2 f01 = unpack_half2(h01), f23 = unpack_half2(h23);
            ls[0] += p0 + p1;
            ls[1] += p2 + p3;
            lrs[0] += f01.x + f01.y;
            lrs[1] += f23.x + f23.y;
            pf[nt >> 1][(nt & 1) * 2 + 0] = h01;
            pf[nt >> 1][(nt & 1) * 2 + 1] = h23;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            ls[e] += __shfl_xor_sync(0xffffffffu, ls[e], 1);
            ls[e] += __shfl_xor_sync(0xffffffffu, ls[e], 2);
            lrs[e] += __shfl_xor_sync(0xffffffffu, lrs[e], 1);
            lrs[e] += __shfl_xor_sync(0xffffffffu, lrs[e], 2);
            l[e] += ls[e];
            lr[e] += lrs[e];
        }
#pragma unroll
        for (int dt = 0; dt < 16; ++dt) {
            oacc[dt][0] *= alpha[0];
            oacc[dt][1] *= alpha[0];
            oacc[dt][2] *= alpha[1];
            oacc[dt][3] *= alpha[1];
        }
        // O += P V
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
            // pf[kc] holds {n-tile 2kc rows g / g+8, n-tile 2kc+1 rows g / g+8}; reorder to A layout
            const uint32_t af[4] = {pf[kc][0], pf[kc][1], pf[kc][2], pf[kc][3]};
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {   // pairs of 8-wide d tiles
                uint32_t bf[4];
                const int r = 16 * kc + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int c = 16 * dp + 8 * (lane >> 4);
                ldmatrix_x4_t(bf, smem_addr(Vb + swz(r, c)));
                mma16816(oacc[2 * dp], af, bf[0], bf[1]);
                mma16816(oacc[2 * dp + 1], af, bf[2], bf[3]);
            }
        }
    }

    // epilogue: O / l_rounded -> fp16 via shared memory; window-row LSE
    __syncthreads();
    const float inv0 = 1.f / lr[0], inv1 = 1.f / lr[1];
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
        const int rr = 16 * warp + g;
        const int c = 8 * dt + 2 * t;
        *reinterpret_cast<uint32_t *>(sQ + swz(rr, c)) = pack_half2(oacc[dt][0] * inv0, oacc[dt][1] * inv0);
        *reinterpret_cast<uint32_t *>(sQ + swz(rr + 8, c)) = pack_half2(oacc[dt][2] * inv1, oacc[dt][3] * inv1);
    }
    if (t == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int row = row_g + 8 * e;
            if (row < a.T && row >= a.T - a.W)
                a.lse2[(size_t)bh * a.W + (row - (a.T - a.W))] = m[e] + log2f(l[e]);
        }
    }
    __syncthreads();
    uint16_t *og = a.o + (size_t)bh * a.T * kD;
    for (int e = tid; e < kBM * 16; e += 128) {
        const int r = e >> 4, ch = e & 15;
        if (q0 + r < a.T)
            *reinterpret_cast<uint4 *>(og + (size_t)(q0 + r) * kD + ch * 8) =
                *reinterpret_cast<const uint4 *>(sQ + swz(r, ch * 8));
    }
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
    extern __shared__ __align__(128) unsigned char smem_raw[];
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

bool g_attr_fa = false;
size_t g_attr_score = 0;

}  // namespace

size_t prefill_workspace_bytes(int B, int Hq, int W) { return ((size_t)B * Hq * W * 4 + 255) / 256 * 256; }

int prefill_launch(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int Hq, int Hkv, int T, int W,
                   float sm_scale, uint16_t *o, float *scores, void *ws, cudaStream_t stream) {
    FaArgs fa;
    fa.q = q; fa.k = k; fa.v = v; fa.o = o;
    fa.lse2 = static_cast<float *>(ws);
    fa.Hq = Hq; fa.Hkv = Hkv; fa.T = T; fa.W = W;
    fa.scale_log2 = sm_scale * kLog2e;
    const size_t fa_smem = (size_t)(kBM + 4 * kBN) * kD * 2;
    if (!g_attr_fa) {
        if (cudaFuncSetAttribute(fa_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fa_smem) !=
            cudaSuccess)
            return check_launch("select_prefill: attribute");
        g_attr_fa = true;
    }
    const int nqt = (T + kBM - 1) / kBM;
    fa_fwd_kernel<<<dim3(nqt, B * Hq), 128, fa_smem, stream>>>(fa);
    int rc = check_launch("select_prefill: flash attention");
    if (rc) return rc;

    ScoreArgs sa;
    sa.q = q; sa.k = k; sa.lse2 = fa.lse2; sa.scores = scores;
    sa.Hq = Hq; sa.Hkv = Hkv; sa.T = T; sa.W = W;
    sa.scale_log2 = fa.scale_log2;
    const int nrows8 = ((Hq / Hkv) * W + 7) / 8 * 8;
    const size_t sc_smem = (size_t)kBN * kD * 2 + (size_t)nrows8 * kD * 2 + (size_t)nrows8 * 4;
    if (sc_smem > g_attr_score) {
        if (cudaFuncSetAttribute(window_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc_smem) !=
            cudaSuccess)
            return check_launch("select_prefill: attribute");
        g_attr_score = sc_smem;
    }
    window_score_kernel<<<dim3((T + kBN - 1) / kBN, B * Hkv), 128, sc_smem, stream>>>(sa);
    return check_launch("select_prefill: window scores");
}

}  // namespace minikv
