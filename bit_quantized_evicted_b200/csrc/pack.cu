// minikv_quant_pack: quantize a compacted kept sequence into the 2-bit cache.
//
// Source: gptget.net summary of arXiv 2411.18077, section 方法论 / 方法详解:
// sub-channel (per-channel) key quantization and per-token value quantization
// into a compact layout.  The newest r tokens stay fp16 in the residual ring.
//
// Traffic: 512 B read and 84 B written per packed token and KV head.  The
// group packer streams it at about half the HBM rate; its limit is instruction
// issue (about 8 instructions per quantized element).
//
// G = 32 or 64: pack_groups_kernel.  Each 128-thread block loops over key
// groups (unit, group) with a stride of the grid, double-buffered: while it
// quantizes one group from shared memory, the G key rows and G value rows of
// its next group are in flight (cp.async into a swizzled tile).  The blocks
// past the group workers copy residual tokens into ring slots 0..r-1.
// G = 128: pack_kernel, one block per (group, unit), reading its rows straight
// from global memory (a staged 128-token tile would leave one block per SM).
//
// minikv_evict_pack runs the same kernels with an index list: compacted token
// t of a unit is then prompt row idx[t] (the kept positions of
// minikv_topk_evict), read straight from the prompt K/V, so the kept rows are
// never written out in fp16 (the fused select -> gather -> pack of the path).
#include <mutex>

#include "common.cuh"

namespace minikv {

namespace {

struct PackArgs {
    const uint16_t *k, *v;
    const int32_t *idx;   // null: rows are contiguous [unit][N]; else row t = prompt row idx[unit][t] of T
    int T;
    uint32_t *k_codes, *v_codes;
    uint16_t *k_scale, *k_zero, *v_scale, *v_zero;
    uint16_t *k_res, *v_res;
    int N, n_q, r, G, Gv, cap, ring, n_groups;
    int unit0;   // cache unit of grid row 0 (b * Hkv when one sequence of a ragged batch is loaded)
    int *dseq;   // device-state mode: [B][4] state words to set (rows seq0 .. seq0 + n_seq - 1), else null
    int seq0, n_seq;
    int units;          // source units (grid rows of pack_kernel)
    int n_work;         // pack_groups_kernel: blocks that pack key groups (the rest copy residual tokens)
    int n_res_blocks;   // residual blocks per unit
};

constexpr int kResPerBlock = 32;   // residual tokens copied per block

__global__ void __launch_bounds__(128) pack_kernel(const PackArgs a) {
    const int src_unit = blockIdx.y;           // unit of the source tensors
    const int unit = a.unit0 + blockIdx.y;     // unit of the cache
    const size_t rows = a.idx ? (size_t)a.T : (size_t)a.N;
    const uint16_t *ku = a.k + (size_t)src_unit * rows * kD;
    const uint16_t *vu = a.v + (size_t)src_unit * rows * kD;
    const int32_t *iu = a.idx ? a.idx + (size_t)src_unit * a.N : nullptr;
    auto src_row = [&](int t) -> size_t { return iu ? (size_t)iu[t] : (size_t)t; };   // compacted -> source row
    if (a.dseq && blockIdx.x == 0 && blockIdx.y == 0)
        for (int b = threadIdx.x; b < a.n_seq; b += 128)
            reinterpret_cast<int4 *>(a.dseq)[a.seq0 + b] = make_int4(a.n_q, a.r, 0, 0);
    if ((int)blockIdx.x < a.n_groups) {
        const int grp = blockIdx.x;
        const int t0 = grp * a.G;
        const size_t tok = (size_t)unit * a.cap + t0;
        const size_t grow = (size_t)unit * (a.cap / a.G) + grp;
        __shared__ float scr[512];
        auto krow = [&](int t, int c) { return ku + src_row(t0 + t) * kD + c; };
        auto vrow = [&](int t, int c) { return vu + src_row(t0 + t) * kD + c; };
        pack_key_group(krow, a.G, a.k_codes + tok * 8, a.k_scale + grow * kD, a.k_zero + grow * kD, scr);
        pack_value_tokens(vrow, a.G, a.Gv, a.v_codes + tok * 8, a.v_scale + tok * (kD / a.Gv),
                          a.v_zero + tok * (kD / a.Gv));
    } else {
        const int i0 = ((int)blockIdx.x - a.n_groups) * kResPerBlock;
        // 16 x 16-byte chunks per token row; 128 threads copy 8 rows per pass
        for (int e = threadIdx.x; e < kResPerBlock * 16; e += 128) {
            const int i = i0 + e / 16, ch = e % 16;
            if (i >= a.r) break;
            const size_t src = src_row(a.n_q + i) * kD;
            const size_t dst = ((size_t)unit * a.ring + i) * kD;
            reinterpret_cast<uint4 *>(a.k_res + dst)[ch] = reinterpret_cast<const uint4 *>(ku + src)[ch];
            reinterpret_cast<uint4 *>(a.v_res + dst)[ch] = reinterpret_cast<const uint4 *>(vu + src)[ch];
        }
    }
}

// ---- pipelined group packer (G = 32 or 64)

constexpr int kPipeThreads = 128;

// fp16x2 word -> its low and high halves as fp32 (exact)
__device__ __forceinline__ void split_h2(uint32_t w, float &lo, float &hi) {
    asm("{\n .reg .f16 l, h;\n mov.b32 {l, h}, %2;\n cvt.f32.f16 %0, l;\n cvt.f32.f16 %1, h;\n}\n"
        : "=f"(lo), "=f"(hi) : "r"(w));
}
// lane-wise min / max of two fp16x2 words (exact, like fminf / fmaxf of the fp32 values)
__device__ __forceinline__ uint32_t hmin2w(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("min.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hmax2w(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// The three comparisons of quant_code_thr on the fp32 FMA pipe.  With
// K = 2^64, fp32 d >= 0 and a threshold t >= 2^-25 or t = +inf,
// sat(fma(d, K, -K t)) is exactly [d > t]: a positive d - t is at least
// ulp(t) >= 2^-48, so K (d - t) >= 2^16, and fma rounds K (d - t) only once;
// a d <= t gives K (d - t) <= 0.  Every nonzero fp16 scale s >= 2^-24 has
// t1, t2, t3 >= 2^-25; s = 0 has infinite thresholds.  [d >= t2] is
// [d > t2'] with t2' the float below t2.
constexpr float kCmpScale = 18446744073709551616.f;   // 2^64
struct QThrK {
    float c1, c2, c3;   // -K t1, -K t2', -K t3
};
__device__ __forceinline__ QThrK scaled_thresholds(const QThr &t) {
    return {-kCmpScale * t.t1, -kCmpScale * __int_as_float(__float_as_int(t.t2) - 1), -kCmpScale * t.t3};
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
// d = fp32(x - zero) for the two fp16 halves of w (low half first): the
// mixed-precision subtraction widens x exactly and rounds once, as
// __fsub_rn(fp32(x), zero) does
__device__ __forceinline__ void sub_h2(uint32_t w, float z0, float z1, float &d0, float &d1) {
    asm("{\n .reg .f16 l, h;\n mov.b32 {l, h}, %2;\n sub.rn.f32.f16 %0, l, %3;\n sub.rn.f32.f16 %1, h, %4;\n}\n"
        : "=f"(d0), "=f"(d1) : "r"(w), "f"(z0), "f"(z1));
}
// w + code(d) * wgt, with code(d) that of quant_code_thr for d = fp32(x - zero)
// and the scaled thresholds of x's channel or block.  w and wgt are small
// integers (wgt a power of 4, at most 8 codes per sum: below 2^16), so every
// step is exact.
__device__ __forceinline__ float add_code_d(float w, float d, float c1, float c2, float c3, float wgt) {
    w = fmaf(fma_sat(d, kCmpScale, c1), wgt, w);
    w = fmaf(fma_sat(d, kCmpScale, c2), wgt, w);
    return fmaf(fma_sat(d, kCmpScale, c3), wgt, w);
}
// codes summed from 2^23 (so the integer sits in the low mantissa bits) -> the code bits
__device__ __forceinline__ uint32_t code_bits(float w) { return (uint32_t)__float_as_int(w) - 0x4B000000u; }
constexpr float kCodeBase = 8388608.f;   // 2^23
__device__ __forceinline__ uint32_t w4(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// One key group from a staged [G][128] tile (swizzled by swz): per channel
// zero = min and scale = (max - min) / 3 over the G tokens, then 2-bit codes.
// Thread (warp w, lane l) takes channels 8q .. 8q+7, q = 4w + l/8, of tokens
// s, s + 8, .. (s = l % 8): min / max in fp16 over its tokens, then over the 8
// slices by xor-shuffles; lane s then sets up channel 8q + s.  Lanes q and
// q ^ 1 hold the two halves of a code word.
template <int G>
__device__ __forceinline__ void pack_keys_tile(const uint16_t *kt, uint32_t *codes, uint16_t *scale_out,
                                               uint16_t *zero_out, float (*thr)[kD]) {
    const int lane = threadIdx.x & 31;
    const int s = lane & 7, q = 4 * (threadIdx.x >> 5) + (lane >> 3);
    uint32_t mn[4], mx[4];
    {
        const uint4 v = *reinterpret_cast<const uint4 *>(kt + swz(s, 8 * q));
#pragma unroll
        for (int i = 0; i < 4; ++i) mn[i] = mx[i] = w4(v, i);
    }
#pragma unroll
    for (int j = 1; j < G / 8; ++j) {
        const uint4 v = *reinterpret_cast<const uint4 *>(kt + swz(s + 8 * j, 8 * q));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mn[i] = hmin2w(mn[i], w4(v, i));
            mx[i] = hmax2w(mx[i], w4(v, i));
        }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            mn[i] = hmin2w(mn[i], __shfl_xor_sync(0xffffffffu, mn[i], o));
            mx[i] = hmax2w(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], o));
        }
    {
        const int i = s >> 1;
        const uint32_t wn = i == 0 ? mn[0] : i == 1 ? mn[1] : i == 2 ? mn[2] : mn[3];
        const uint32_t wx = i == 0 ? mx[0] : i == 1 ? mx[1] : i == 2 ? mx[2] : mx[3];
        float nlo, nhi, xlo, xhi;
        split_h2(wn, nlo, nhi);
        split_h2(wx, xlo, xhi);
        const float fmn = canon_zero((s & 1) ? nhi : nlo), fmx = canon_zero((s & 1) ? xhi : xlo);
        const uint16_t sb = quant_scale(fmn, fmx);
        const int c = 8 * q + s;
        scale_out[c] = sb;
        zero_out[c] = f2h(fmn);
        const QThrK th = scaled_thresholds(quant_thresholds(h2f(sb)));
        thr[0][c] = fmn;
        thr[1][c] = th.c1;
        thr[2][c] = th.c2;
        thr[3][c] = th.c3;
    }
    __syncwarp();   // channel 8q + s was set up by lane s of this lane's own group of 8
    float z[8], t1[8], t2[8], t3[8];   // zero and the scaled thresholds c1, c2, c3
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float4 a0 = *reinterpret_cast<const float4 *>(&thr[0][8 * q + 4 * h]);
        const float4 a1 = *reinterpret_cast<const float4 *>(&thr[1][8 * q + 4 * h]);
        const float4 a2 = *reinterpret_cast<const float4 *>(&thr[2][8 * q + 4 * h]);
        const float4 a3 = *reinterpret_cast<const float4 *>(&thr[3][8 * q + 4 * h]);
        z[4 * h] = a0.x; z[4 * h + 1] = a0.y; z[4 * h + 2] = a0.z; z[4 * h + 3] = a0.w;
        t1[4 * h] = a1.x; t1[4 * h + 1] = a1.y; t1[4 * h + 2] = a1.z; t1[4 * h + 3] = a1.w;
        t2[4 * h] = a2.x; t2[4 * h + 1] = a2.y; t2[4 * h + 2] = a2.z; t2[4 * h + 3] = a2.w;
        t3[4 * h] = a3.x; t3[4 * h + 1] = a3.y; t3[4 * h + 2] = a3.z; t3[4 * h + 3] = a3.w;
    }
#pragma unroll
    for (int j = 0; j < G / 8; ++j) {
        const int t = s + 8 * j;
        const uint4 v = *reinterpret_cast<const uint4 *>(kt + swz(t, 8 * q));
        float hw = kCodeBase;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float d0, d1;
            sub_h2(w4(v, i), z[2 * i], z[2 * i + 1], d0, d1);
            hw = add_code_d(hw, d0, t1[2 * i], t2[2 * i], t3[2 * i], (float)(1 << (4 * i)));
            hw = add_code_d(hw, d1, t1[2 * i + 1], t2[2 * i + 1], t3[2 * i + 1], (float)(1 << (4 * i + 2)));
        }
        const uint32_t h = code_bits(hw);
        const uint32_t other = __shfl_xor_sync(0xffffffffu, h, 8);
        if (!(q & 1)) codes[t * 8 + (q >> 1)] = h | (other << 16);
    }
}

// The G value tokens of a staged tile, each quantized per block of Gv
// channels (Gv in {16, 32, 64, 128}): thread 4i + k takes token i (then
// i + 32) and its channels 32k .. 32k+31, as pack_value_tokens does; min / max
// in fp16, combined over the Gv/32 threads of a block wider than 32 channels.
template <int G>
__device__ __forceinline__ void pack_values_tile(const uint16_t *vt, int Gv, uint32_t *codes, uint16_t *scale_out,
                                                 uint16_t *zero_out) {
    const int k = threadIdx.x & 3;
    const int nb = kD / Gv;
#pragma unroll 1
    for (int t = threadIdx.x >> 2; t < G; t += kPipeThreads / 4) {
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(vt + swz(t, 32 * k + 8 * c));
            w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
        }
        float fmn[2], fmx[2];   // per 16-channel half
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t a = w[8 * h], b = w[8 * h];
#pragma unroll
            for (int i = 1; i < 8; ++i) {
                a = hmin2w(a, w[8 * h + i]);
                b = hmax2w(b, w[8 * h + i]);
            }
            float alo, ahi, blo, bhi;
            split_h2(a, alo, ahi);
            split_h2(b, blo, bhi);
            fmn[h] = fminf(alo, ahi);
            fmx[h] = fmaxf(blo, bhi);
        }
        float zh[2], t1[2], t2[2], t3[2];   // zero and the scaled thresholds c1, c2, c3 per half
        if (Gv == 16) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float mn = canon_zero(fmn[h]), mx = canon_zero(fmx[h]);
                const uint16_t sb = quant_scale(mn, mx);
                scale_out[t * nb + 2 * k + h] = sb;
                zero_out[t * nb + 2 * k + h] = f2h(mn);
                const QThrK th = scaled_thresholds(quant_thresholds(h2f(sb)));
                zh[h] = mn;
                t1[h] = th.c1;
                t2[h] = th.c2;
                t3[h] = th.c3;
            }
        } else {
            float mn = fminf(fmn[0], fmn[1]), mx = fmaxf(fmx[0], fmx[1]);
            for (int o = 1; o < Gv / 32; o <<= 1) {   // the threads of one token are adjacent lanes
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            mn = canon_zero(mn);
            mx = canon_zero(mx);
            const uint16_t sb = quant_scale(mn, mx);
            const int per = Gv / 32;   // threads per block
            if ((k % per) == 0) {
                scale_out[t * nb + k / per] = sb;
                zero_out[t * nb + k / per] = f2h(mn);
            }
            const QThrK th = scaled_thresholds(quant_thresholds(h2f(sb)));
            zh[0] = zh[1] = mn;
            t1[0] = t1[1] = th.c1;
            t2[0] = t2[1] = th.c2;
            t3[0] = t3[1] = th.c3;
        }
        uint32_t cw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float c[2] = {kCodeBase, kCodeBase};   // the word's low and high 16 bits (8 channels each)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float d0, d1;
                sub_h2(w[8 * h + i], zh[h], zh[h], d0, d1);
                const int j = i & 3;
                c[i >> 2] = add_code_d(c[i >> 2], d0, t1[h], t2[h], t3[h], (float)(1 << (4 * j)));
                c[i >> 2] = add_code_d(c[i >> 2], d1, t1[h], t2[h], t3[h], (float)(1 << (4 * j + 2)));
            }
            cw[h] = code_bits(c[0]) | (code_bits(c[1]) << 16);
        }
        *reinterpret_cast<uint2 *>(codes + t * 8 + 2 * k) = make_uint2(cw[0], cw[1]);
    }
}

// Blocks 0 .. n_work-1 pack key groups (task = source unit * n_groups + group,
// strided by n_work, the next task's rows in flight while one is packed); the
// blocks after them copy residual tokens, n_res_blocks per unit.
template <int G>
__global__ void __launch_bounds__(kPipeThreads) pack_groups_kernel(const PackArgs a) {
    extern __shared__ __align__(16) uint16_t tiles[];   // [2][K tile, V tile], each [G][128] swizzled
    __shared__ __align__(16) float thr[4][kD];          // per key channel: zero, t1, t2, t3
    const int tid = threadIdx.x;
    const size_t rows = a.idx ? (size_t)a.T : (size_t)a.N;
    if (a.dseq && blockIdx.x == 0)
        for (int b = tid; b < a.n_seq; b += kPipeThreads)
            reinterpret_cast<int4 *>(a.dseq)[a.seq0 + b] = make_int4(a.n_q, a.r, 0, 0);
    if ((int)blockIdx.x < a.n_work) {
        const int n_tasks = a.units * a.n_groups;
        auto issue = [&](int task, int buf) {
            if (task < n_tasks) {
                const int su = task / a.n_groups, grp = task - su * a.n_groups;
                const uint16_t *ku = a.k + (size_t)su * rows * kD, *vu = a.v + (size_t)su * rows * kD;
                const int32_t *iu = a.idx ? a.idx + (size_t)su * a.N : nullptr;
                uint16_t *kt = tiles + buf * (2 * G * kD), *vt = kt + G * kD;
                for (int e = tid; e < G * 16; e += kPipeThreads) {
                    const int t = e >> 4, ch = e & 15, tt = grp * G + t;
                    const size_t src = (iu ? (size_t)iu[tt] : (size_t)tt) * kD + ch * 8;
                    cp_async16(smem_addr(kt + swz(t, ch * 8)), ku + src, true);
                    cp_async16(smem_addr(vt + swz(t, ch * 8)), vu + src, true);
                }
            }
            cp_async_commit();
        };
        int buf = 0;
        issue(blockIdx.x, 0);
        for (int task = blockIdx.x; task < n_tasks; task += a.n_work, buf ^= 1) {
            issue(task + a.n_work, buf ^ 1);
            cp_async_wait<1>();
            __syncthreads();
            const int su = task / a.n_groups, grp = task - su * a.n_groups;
            const int unit = a.unit0 + su;
            const size_t tok = (size_t)unit * a.cap + (size_t)grp * G;
            const size_t grow = (size_t)unit * (a.cap / G) + grp;
            const uint16_t *kt = tiles + buf * (2 * G * kD), *vt = kt + G * kD;
            pack_keys_tile<G>(kt, a.k_codes + tok * 8, a.k_scale + grow * kD, a.k_zero + grow * kD, thr);
            pack_values_tile<G>(vt, a.Gv, a.v_codes + tok * 8, a.v_scale + tok * (kD / a.Gv),
                                a.v_zero + tok * (kD / a.Gv));
            __syncthreads();   // this tile and thr are free for the group after next
        }
        cp_async_wait<0>();
        return;
    }
    // residual tokens: block (unit su, part rb) copies tokens 32 rb .. 32 rb + 31
    const int rblk = (int)blockIdx.x - a.n_work;
    if (a.n_res_blocks == 0) return;
    const int su = rblk / a.n_res_blocks, rb = rblk - su * a.n_res_blocks;
    if (su >= a.units) return;
    const int unit = a.unit0 + su;
    const uint16_t *ku = a.k + (size_t)su * rows * kD, *vu = a.v + (size_t)su * rows * kD;
    const int32_t *iu = a.idx ? a.idx + (size_t)su * a.N : nullptr;
    const int i0 = rb * kResPerBlock;
    for (int e = tid; e < kResPerBlock * 16; e += kPipeThreads) {
        const int i = i0 + e / 16, ch = e % 16;
        if (i >= a.r) break;
        const int tt = a.n_q + i;
        const size_t src = (iu ? (size_t)iu[tt] : (size_t)tt) * kD;
        const size_t dst = ((size_t)unit * a.ring + i) * kD;
        reinterpret_cast<uint4 *>(a.k_res + dst)[ch] = reinterpret_cast<const uint4 *>(ku + src)[ch];
        reinterpret_cast<uint4 *>(a.v_res + dst)[ch] = reinterpret_cast<const uint4 *>(vu + src)[ch];
    }
}

// Resident blocks of pack_groups_kernel<G> on device dev (one-time set-up per
// device: the shared-memory opt-in and the occupancy query); 0 on a CUDA error.
std::mutex g_pack_mu;
int g_pack_slots[kMaxDevices][2] = {};

template <int G>
int pack_slots(int dev) {
    std::lock_guard<std::mutex> lk(g_pack_mu);
    int &slots = g_pack_slots[dev][G == 64];
    if (slots > 0) return slots;
    const int smem = 2 * 2 * G * kD * (int)sizeof(uint16_t);
    int per_sm = 0, sms = 0;
    if (cudaFuncSetAttribute(pack_groups_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pack_groups_kernel<G>, kPipeThreads, smem) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || per_sm < 1 || sms < 1)
        return 0;
    slots = per_sm * sms;
    return slots;
}

}  // namespace

// idx == nullptr: k, v are [B,Hkv,N,D]; else k, v are [B,Hkv,T,D] and row t of
// unit u is idx[u][t] (idx [B,Hkv,N], ascending positions < T).  seq >= 0 loads
// sequence `seq` of a ragged cache only (k, v, idx then without the B axis).
// With a device-state cache, block (0, 0) also writes the loaded rows' state.
int pack_launch(minikv_cache *c, const uint16_t *k, const uint16_t *v, int N, cudaStream_t stream,
                const int32_t *idx, int T, int seq) {
    int n_q, r;
    if (N >= c->R) {
        r = c->R + (N - c->R) % c->G;
        n_q = N - r;
    } else {
        r = N;
        n_q = 0;
    }
    if (n_q > c->cap)
        return fail(MINIKV_ERR_CAPACITY, "quant_pack: %d packed tokens exceed cap=%d", n_q, c->cap);
    PackArgs a;
    a.k = k; a.v = v;
    a.idx = idx; a.T = T;
    a.k_codes = c->k_codes; a.v_codes = c->v_codes;
    a.k_scale = c->k_scale; a.k_zero = c->k_zero; a.v_scale = c->v_scale; a.v_zero = c->v_zero;
    a.k_res = c->k_res; a.v_res = c->v_res;
    a.N = N; a.n_q = n_q; a.r = r; a.G = c->G; a.Gv = c->Gv; a.cap = c->cap; a.ring = c->R + c->G;
    a.n_groups = n_q / c->G;
    a.unit0 = seq >= 0 ? seq * c->Hkv : 0;
    a.dseq = c->dseq;
    a.seq0 = seq >= 0 ? seq : 0;
    a.n_seq = seq >= 0 ? 1 : c->B;
    const int n_res_blocks = (r + kResPerBlock - 1) / kResPerBlock;
    const int units = seq >= 0 ? c->Hkv : c->B * c->Hkv;
    a.units = units;
    a.n_res_blocks = n_res_blocks;
    a.n_work = 0;
    if (c->G <= 64) {
        const int dev = current_device();
        if (dev < 0) return fail(MINIKV_ERR_CUDA, "quant_pack: no current CUDA device");
        const int slots = c->G == 32 ? pack_slots<32>(dev) : pack_slots<64>(dev);
        if (slots < 1) {
            const int rc = check_launch("quant_pack: set-up");
            return rc ? rc : fail(MINIKV_ERR_CUDA, "quant_pack: no resident block of the pack kernel");
        }
        const long long n_tasks = (long long)units * a.n_groups;
        a.n_work = (int)(n_tasks < slots ? n_tasks : slots);
        long long grid = a.n_work + (long long)n_res_blocks * units;
        if (c->dseq && grid == 0) grid = 1;   // an empty load still sets the device state
        if (grid > 0) {
            const size_t smem = (size_t)2 * 2 * c->G * kD * sizeof(uint16_t);
            if (c->G == 32) pack_groups_kernel<32><<<(unsigned)grid, kPipeThreads, smem, stream>>>(a);
            else pack_groups_kernel<64><<<(unsigned)grid, kPipeThreads, smem, stream>>>(a);
            const int rc = check_launch("quant_pack");
            if (rc) return rc;
        }
    } else {
        int gx = a.n_groups + n_res_blocks;
        if (c->dseq && gx == 0) gx = 1;   // an empty load still sets the device state
        if (gx > 0 && units > 0) {
            pack_kernel<<<dim3(gx, units), 128, 0, stream>>>(a);
            const int rc = check_launch("quant_pack");
            if (rc) return rc;
        }
    }
    if (seq >= 0) {
        if (c->seq) {
            c->seq[3 * seq] = n_q;
            c->seq[3 * seq + 1] = r;
            c->seq[3 * seq + 2] = 0;
        }
        return MINIKV_OK;
    }
    c->n_packed = n_q;
    c->n_res = r;
    c->res_start = 0;
    if (c->seq)
        for (int b = 0; b < c->B; ++b) {
            c->seq[3 * b] = n_q;
            c->seq[3 * b + 1] = r;
            c->seq[3 * b + 2] = 0;
        }
    return MINIKV_OK;
}

}  // namespace minikv
