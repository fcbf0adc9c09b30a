// Shared device helpers of libminikv (sm_100a).
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/minikv.h"

namespace minikv {

// Host-side error reporting (minikv_api.cu).  Returns `code`.
int fail(int code, const char *fmt, ...);
int check_launch(const char *what);

constexpr int kD = 128;                  // the one supported head size
constexpr int kMaxDevices = 64;          // device ordinals of the per-device set-up caches

// The current device's ordinal, or -1 if it cannot be read or is not below
// kMaxDevices (host code; per-device caches are indexed by it).
inline int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float h2f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ uint16_t f2h(float f) { return __half_as_ushort(__float2half_rn(f)); }

// Two floats -> half2 bits (lo in bits 0..15), round to nearest even.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float2 unpack_half2(uint32_t x) {
    __half2 h = *reinterpret_cast<__half2 *>(&x);
    return __half22float2(h);
}

// Packed fp32 pairs (lo in bits 0..31): one f32x2 instruction per two lanes of work.
__device__ __forceinline__ unsigned long long f2pack(float lo, float hi) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};\n" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long x, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;\n" : "=f"(lo), "=f"(hi) : "l"(x));
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long fmul2(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// D (16x8 fp32) += A (16x16 fp16, row) * B (16x8 fp16, col).
// Fragment ownership, g = lane/4, t = lane%4:
//   A: a[0]={(g,2t),(g,2t+1)} a[1]={(g+8,2t),(g+8,2t+1)} a[2]={(g,2t+8),(g,2t+9)} a[3]={(g+8,2t+8),(g+8,2t+9)}
//   B: b[0]={(2t,g),(2t+1,g)} b[1]={(2t+8,g),(2t+9,g)}       (k, n)
//   D: d[0]=(g,2t) d[1]=(g,2t+1) d[2]=(g+8,2t) d[3]=(g+8,2t+1)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held one row-pair per thread: in, thread (g,t)
// holds (row g, cols 2t..2t+1); out, it holds (row g, cols 2t..2t+1) of the transpose.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(saddr));
}
__device__ __forceinline__ void ldmatrix_x4_t(uint32_t (&r)[4], uint32_t saddr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(saddr));
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy (Ampere-style cp.async), zero-filled when !pred.
__device__ __forceinline__ void cp_async16(uint32_t saddr, const void *g, bool pred) {
    int n = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// ---- mbarriers ----------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
// Wait for phase `parity` of the barrier to complete.  Bounded: gives up after
// ~`limit` polls and returns false, so a lost transfer can never hang the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t limit = (1u << 26)) {
    uint32_t addr = smem_addr(bar);
    for (uint32_t i = 0; i < limit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done) : "r"(addr), "r"(parity) : "memory");
        if (done) return true;
    }
    return false;
}
// ---- the 2-bit quantizer (bit-exact: one IEEE fp32 op per step) -------------

// scale = fp16_rn(fp32(mx - mn) / 3); mn/mx already canonical (+0 for zero).
__device__ __forceinline__ uint16_t quant_scale(float mn, float mx) {
    return f2h(__fdiv_rn(__fsub_rn(mx, mn), 3.0f));
}
// code = clamp(rint((x - zero) / scale), 0, 3), 0 when scale == 0: the
// definition; the pack helpers compute it as quant_code_thr below.
__device__ __forceinline__ uint32_t quant_code(float x, float zero, float scale) {
    if (scale == 0.0f) return 0u;
    float q = rintf(__fdiv_rn(__fsub_rn(x, zero), scale));
    q = fminf(fmaxf(q, 0.0f), 3.0f);
    return static_cast<uint32_t>(q);
}
// The same code without a division.  With d = fp32(x - zero) >= 0 and s > 0,
// rint(RN(d / s)) is decided by where the exact quotient d/s lies against the
// rounding boundaries of RN at 0.5, 1.5 and 2.5 (ties to even):
//   code >= 1  <=>  RN(d/s) >  0.5  <=>  d/s >  0.5 + 2^-25
//   code >= 2  <=>  RN(d/s) >= 1.5  <=>  d/s >= 1.5 - 2^-24
//   code >= 3  <=>  RN(d/s) >  2.5  <=>  d/s >  2.5 + 2^-23
// Each boundary times s is exact in fp64 (at most 25 x 24 significant bits);
// rounding it down (for >) or up (for >=) to fp32 gives a threshold that an
// fp32 d can be compared with exactly.  s == 0 gives code 0 everywhere.
struct QThr {
    float t1, t2, t3;
};
__device__ __forceinline__ QThr quant_thresholds(float s) {
    if (s == 0.0f) return {INFINITY, INFINITY, INFINITY};
    const double sd = (double)s;
    return {__double2float_rd(sd * (0.5 + 0x1p-25)), __double2float_ru(sd * (1.5 - 0x1p-24)),
            __double2float_rd(sd * (2.5 + 0x1p-23))};
}
__device__ __forceinline__ uint32_t quant_code_thr(float x, float zero, const QThr &t) {
    const float d = __fsub_rn(x, zero);
    return (uint32_t)(d > t.t1) + (uint32_t)(d >= t.t2) + (uint32_t)(d > t.t3);
}
// -0 and +0 are the same extreme; store +0.
__device__ __forceinline__ float canon_zero(float x) { return __fadd_rn(x, 0.0f); }

// element offset of (row, col) in a [rows][128] fp16 tile; 16-byte chunks are
// XOR-swizzled by row so ldmatrix reads of 8 rows, and column reads of one
// row by a warp, hit distinct banks
__device__ __forceinline__ int swz(int row, int col) {
    return row * kD + ((((col >> 3) ^ (row & 7))) << 3) + (col & 7);
}

// fp16 bits -> float, 8 at a time (one 16-byte chunk)
__device__ __forceinline__ void h8_to_f(uint4 v, float *x) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = h2f((uint16_t)(w[i] & 0xffffu));
        x[2 * i + 1] = h2f((uint16_t)(w[i] >> 16));
    }
}

// Pack one key group: G tokens x 128 channels -> codes (token-major words),
// one (scale, zero) per channel.  Called by all NT threads of a CTA (NT a
// multiple of 128; threads 0..127 take one channel each in step 1).
// at(t, c) points to channel c of token t (global or shared memory); the 8
// channels of each aligned 8-channel chunk are contiguous and 16-byte aligned.
// scr: 512 floats of shared scratch.
//   1. thread c: min / max of channel c over the G tokens -> (zero, scale);
//   2. thread i: code words i, i + 128, ... (token w / 8, channels 16 (w % 8)
//      .. +15), each from two 16-byte loads and 16 independent quantizations.
template <int NT = 128, class AtFn>
__device__ __forceinline__ void pack_key_group(AtFn at, int G, uint32_t *codes /* [G][8] */,
                                               uint16_t *scale_out /* [128] */, uint16_t *zero_out,
                                               float *scr /* [512] shared */) {
    const int c = threadIdx.x;
    if (c < kD) {
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll 8
        for (int t = 0; t < G; ++t) {
            const float x = h2f(*at(t, c));
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
        }
        mn = canon_zero(mn);
        mx = canon_zero(mx);
        const uint16_t sb = quant_scale(mn, mx);
        scale_out[c] = sb;
        zero_out[c] = f2h(mn);
        const QThr th = quant_thresholds(h2f(sb));
        scr[c] = mn;
        scr[128 + c] = th.t1;
        scr[256 + c] = th.t2;
        scr[384 + c] = th.t3;
    }
    __syncthreads();
    for (int wi = c; wi < G * 8; wi += NT) {
        const int t = wi >> 3, c0 = 16 * (wi & 7);
        float x[16];
        h8_to_f(*reinterpret_cast<const uint4 *>(at(t, c0)), x);
        h8_to_f(*reinterpret_cast<const uint4 *>(at(t, c0 + 8)), x + 8);
        uint32_t w = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const QThr t = {scr[128 + c0 + i], scr[256 + c0 + i], scr[384 + c0 + i]};
            w |= quant_code_thr(x[i], scr[c0 + i], t) << (2 * i);
        }
        codes[wi] = w;
    }
    __syncthreads();   // scr is free again
}

// Pack value tokens: each of n tokens is quantized per block of Gv channels.
// Called by all NT threads: thread 4j + k of a pass takes token (pass * NT/4 + j)
// and its channels 32k .. 32k+31 (two code words); min / max of a block wider
// than 32 channels are combined over the Gv/32 threads that share it.
// Gv in {16, 32, 64, 128}.  at() as for pack_key_group.
template <int NT = 128, class AtFn>
__device__ __forceinline__ void pack_value_tokens(AtFn at, int n, int Gv, uint32_t *codes /* [n][8] */,
                                                  uint16_t *scale_out /* [n][128/Gv] */, uint16_t *zero_out) {
    const int k = threadIdx.x & 3;
    const int nb = kD / Gv;   // blocks per token
    for (int t0 = 0; t0 < n; t0 += NT / 4) {
        const int t = t0 + (threadIdx.x >> 2);
        const bool live = t < n;
        float x[32];
        if (live) {
#pragma unroll
            for (int q = 0; q < 4; ++q) h8_to_f(*reinterpret_cast<const uint4 *>(at(t, 32 * k + 8 * q)), x + 8 * q);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = 0.f;
        }
        // (mn, s) of the block(s) these 32 channels fall in: halves h = 0, 1 (16 channels each)
        float mnh[2];
        QThr th[2];
        if (Gv == 16) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float mn = x[16 * h], mx = x[16 * h];
#pragma unroll
                for (int i = 1; i < 16; ++i) {
                    mn = fminf(mn, x[16 * h + i]);
                    mx = fmaxf(mx, x[16 * h + i]);
                }
                mn = canon_zero(mn);
                mx = canon_zero(mx);
                const uint16_t sb = quant_scale(mn, mx);
                if (live) {
                    scale_out[t * nb + 2 * k + h] = sb;
                    zero_out[t * nb + 2 * k + h] = f2h(mn);
                }
                mnh[h] = mn;
                th[h] = quant_thresholds(h2f(sb));
            }
        } else {
            float mn = x[0], mx = x[0];
#pragma unroll
            for (int i = 1; i < 32; ++i) {
                mn = fminf(mn, x[i]);
                mx = fmaxf(mx, x[i]);
            }
            for (int o = 1; o < Gv / 32; o <<= 1) {   // the threads of one token are adjacent lanes
                mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            }
            mn = canon_zero(mn);
            mx = canon_zero(mx);
            const uint16_t sb = quant_scale(mn, mx);
            const int per = Gv / 32;   // threads per block
            if (live && (k % per) == 0) {
                scale_out[t * nb + k / per] = sb;
                zero_out[t * nb + k / per] = f2h(mn);
            }
            mnh[0] = mnh[1] = mn;
            th[0] = th[1] = quant_thresholds(h2f(sb));
        }
        if (live) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 16; ++i) w |= quant_code_thr(x[16 * h + i], mnh[h], th[h]) << (2 * i);
                codes[t * 8 + 2 * k + h] = w;
            }
        }
    }
}

}  // namespace minikv
