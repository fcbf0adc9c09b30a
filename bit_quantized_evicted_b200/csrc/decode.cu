// minikv_decode_attn: one decoding step over the 2-bit cache (flash-decoding).
//
// Source: MiniKV abstract (specialized CUDA kernels compatible with
// FlashAttention) and the gptget.net summary of arXiv 2411.18077, section
// 方法论 (sub-channel key / per-token value 2-bit quantization, compact layout).
//
// One launch per layer-step, one CTA of 4 warps per work item:
//   * residual CTAs, n_rc per (sequence, KV head) "unit": 64-token chunks of the
//     fp16 residual ring, staged by cp.async into swizzled shared memory; the
//     chunk holding the new token appends it to the ring, chunk 0 packs the
//     oldest G tokens to 2 bits when the residual is full (same code as
//     minikv_quant_pack);
//   * packed CTAs, sized to fill the GPU once: the packed tokens of all units,
//     cut into 32-token slices, are laid end to end and split evenly into P
//     contiguous ranges (one per CTA).  Each warp owns a 4-stage TMA-bulk
//     pipeline (cp.async.bulk + mbarrier) over its slices of the range.
// Every CTA writes one partial softmax state (m, l, sum p*v) per unit it
// touched; the last CTA to arrive at a unit (self-resetting atomic counter)
// merges them into `out`.
//
// Slice math (per warp, 32 tokens = 2 m-tiles of 16, g <= 4 query heads):
//   codes -> fp16 SUBNORMALS: one AND puts a 2-bit code at mantissa bit p in
//     {4, 6, 8} of both halves of a 32-bit word, i.e. the value code * 2^(p-24)
//     (mma.sync consumes fp16 subnormals exactly);
//   scores  S[tok, col] = sum_c code_c 2^(p_c-24) b_c,   b_c = q_c s_c 2^(8-p_c)
//     split hi + lo in fp16 (HMUL2 / HFMA2): columns 0..3 hold the hi parts of
//     heads 0..3, columns 4..7 the lo parts; the accumulator starts at the
//     zero-point term sum_c q_c z_c, itself one mma per 16 channels (A = the
//     key-zero row broadcast to all 16 rows, B = q);
//   output  O^T[ch, col] = sum_t code_{t,ch} 2^(p-24) P'[t, col],  P' = p_t * v_scale_t
//     (hi/lo), moved from the score fragment layout into the B layout by
//     movmatrix; out_ch = (O^T[ch,h] + O^T[ch,h+4]) 2^(24-p) + sum_t p_t v_zero_t.
// A 16-token m-tile takes its tokens in the order perm8 so that both the
// key-word and the value-word shared loads of a warp hit 32 distinct banks.
//
// Attention-mass variant (decode_kernel<true>, minikv_decode_attn_mass): every
// CTA also stores the absolute log2 score of each token it scores, per query
// head, into a workspace array; the merging CTA of a unit stores the unit's
// final (max, sum) per head; mass_kernel then adds
// sum_h 2^(x_h,t - M_h) / L_h to the caller's running score of token t, the
// H2O-style accumulated attention the MiniKV summary's experiments compare with.
#include <math.h>

#include "common.cuh"

namespace minikv {

namespace {

constexpr int kThreads = 128;
constexpr int kSlice = 32;         // packed tokens per warp work item
constexpr int kWarpStages = 4;
constexpr int kResChunk = 64;      // residual tokens per residual CTA
constexpr int kPartStride = 132;   // floats per (unit, slot, head): y[128], m, l
constexpr int kMaxPackedCtas = 4096;

struct __align__(16) SliceBuf {
    uint32_t kc[kSlice * 8];   // key codes, token-major
    uint32_t vc[kSlice * 8];   // value codes
    uint16_t ks[kD];           // key scales of the slice's group
    uint16_t kz[kD];           // key zeros of the slice's group
    uint16_t vs[kSlice];       // value scales
    uint16_t vz[kSlice];       // value zeros
};
constexpr uint32_t kSliceBytes = sizeof(SliceBuf);
static_assert(kSliceBytes == 2688, "slice buffer layout");

struct __align__(16) Smem {
    union {
        SliceBuf st[4][kWarpStages];
        struct {
            uint16_t k[kResChunk * kD];   // XOR-swizzled rows (see swz)
            uint16_t v[kResChunk * kD];
        } res;
    };
    uint16_t qn[8][kD];      // query rows of the current unit (rows >= g are zero)
    uint64_t full[4][kWarpStages];
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
    unsigned *grid_counter;   // device-state mode: CTAs of this launch that have finished (self-resetting)
    int *dseq;                // device-state mode: per-sequence state [B][4] in device memory
    float *xs;          // mass variant: absolute log2 scores [unit][g][xs_stride]
    float *stats;       // mass variant: per unit max[4], sum[4], token count (int bits), pad
    int xs_stride;
    int Hkv, g, G, cap, ring;
    int n_q, r, res_start, flush;
    int units, n_rc, spu, P, S_max;   // schedule: slices per unit, packed CTAs, partial slots per unit
    int groups_cap, lg2G;             // cap / G and log2(G)
    int Ns;                           // total slices (< 2^31)
    float scale_log2;
};

// Ragged batches: each sequence b has its own packed count, residual count (the
// new token included) and ring origin.  The table travels as a kernel parameter
// (__grid_constant__, read through the constant cache), so a step needs no
// host-to-device copy.  sbeg[b] = first flat slice of sequence b's units.
constexpr int kMaxRaggedSeqs = MINIKV_MAX_RAGGED_SEQS;
struct SeqTab {
    int n_q[kMaxRaggedSeqs];
    int r[kMaxRaggedSeqs];
    int res_start[kMaxRaggedSeqs];
    int sbeg[kMaxRaggedSeqs + 1];
};
struct ArgsVar : Args {
    SeqTab tab;
};

// Per-unit lengths.  Uniform batches read the shared scalars; ragged ones the
// table.  slice0 = the unit's first slice in the flat list of all units'
// packed slices; unit_of = the unit holding flat slice x (x < Ns).
__device__ __forceinline__ int len_nq(const Args &a, int) { return a.n_q; }
__device__ __forceinline__ int len_r(const Args &a, int) { return a.r; }
__device__ __forceinline__ int len_rs(const Args &a, int) { return a.res_start; }
__device__ __forceinline__ int len_spu(const Args &a, int) { return a.spu; }
__device__ __forceinline__ int seq_spu(const Args &a, int) { return a.spu; }
__device__ __forceinline__ int slice0(const Args &a, int unit) { return unit * a.spu; }
__device__ __forceinline__ int unit_of(const Args &a, int x) { return x / a.spu; }

__device__ __forceinline__ int len_nq(const ArgsVar &a, int unit) { return a.tab.n_q[unit / a.Hkv]; }
__device__ __forceinline__ int len_r(const ArgsVar &a, int unit) { return a.tab.r[unit / a.Hkv]; }
__device__ __forceinline__ int len_rs(const ArgsVar &a, int unit) { return a.tab.res_start[unit / a.Hkv]; }
__device__ __forceinline__ int len_spu(const ArgsVar &a, int unit) { return a.tab.n_q[unit / a.Hkv] / kSlice; }
__device__ __forceinline__ int seq_spu(const ArgsVar &a, int b) { return a.tab.n_q[b] / kSlice; }
__device__ __forceinline__ int slice0(const ArgsVar &a, int unit) {
    const int b = unit / a.Hkv;
    return a.tab.sbeg[b] + (unit - b * a.Hkv) * (a.tab.n_q[b] / kSlice);
}
__device__ __forceinline__ int unit_of(const ArgsVar &a, int x) {
    // largest b with sbeg[b] <= x; since x < sbeg[B], sequence b has slices
    int lo = 0, hi = a.units / a.Hkv;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.tab.sbeg[mid] <= x) lo = mid;
        else hi = mid;
    }
    return lo * a.Hkv + (x - a.tab.sbeg[lo]) / (a.tab.n_q[lo] / kSlice);
}

// Device-state mode: the per-sequence state lives in device memory (dseq), so
// one launch configuration serves every step and the calls can be captured in
// a CUDA graph.  Each CTA copies the state into shared memory behind Smem
// (DevTab) before it starts; the partition of the packed slices over the
// packed CTAs is then computed from it, on the device.
struct ArgsDev : Args {};
struct DevTab {   // followed by n_q[B], r[B], res_start[B], sbeg[B + 1]
    int Ns, P;    // packed slices this step, packed CTAs that take a share
};
__device__ __forceinline__ unsigned char *dyn_smem() {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    return smem_raw;
}
__device__ __forceinline__ DevTab &dev_tab() { return *reinterpret_cast<DevTab *>(dyn_smem() + sizeof(Smem)); }
__device__ __forceinline__ int *dev_arr(const ArgsDev &a, int k) {   // k = 0 n_q, 1 r, 2 res_start, 3 sbeg
    return reinterpret_cast<int *>(dyn_smem() + sizeof(Smem) + sizeof(DevTab)) + k * (a.units / a.Hkv);
}
__device__ __forceinline__ int len_nq(const ArgsDev &a, int unit) { return dev_arr(a, 0)[unit / a.Hkv]; }
__device__ __forceinline__ int len_r(const ArgsDev &a, int unit) { return dev_arr(a, 1)[unit / a.Hkv]; }
__device__ __forceinline__ int len_rs(const ArgsDev &a, int unit) { return dev_arr(a, 2)[unit / a.Hkv]; }
__device__ __forceinline__ int len_spu(const ArgsDev &a, int unit) { return dev_arr(a, 0)[unit / a.Hkv] / kSlice; }
__device__ __forceinline__ int seq_spu(const ArgsDev &a, int b) { return dev_arr(a, 0)[b] / kSlice; }
__device__ __forceinline__ int slice0(const ArgsDev &a, int unit) {
    const int b = unit / a.Hkv;
    return dev_arr(a, 3)[b] + (unit - b * a.Hkv) * (dev_arr(a, 0)[b] / kSlice);
}
__device__ __forceinline__ int unit_of(const ArgsDev &a, int x) {
    const int *sbeg = dev_arr(a, 3);
    int lo = 0, hi = a.units / a.Hkv;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (sbeg[mid] <= x) lo = mid;
        else hi = mid;
    }
    return lo * a.Hkv + (x - sbeg[lo]) / (dev_arr(a, 0)[lo] / kSlice);
}

// the partition of packed slices over packed CTAs (host-planned, or this step's on the device)
__device__ __forceinline__ int part_Ns(const Args &a) { return a.Ns; }
__device__ __forceinline__ int part_P(const Args &a) { return a.P; }
__device__ __forceinline__ int part_Ns(const ArgsDev &) { return dev_tab().Ns; }
__device__ __forceinline__ int part_P(const ArgsDev &) { return dev_tab().P; }

// column of element `col` of query row h in the swizzled sm.qn rows
__device__ __forceinline__ int qn_col(int h, int col) { return (((col >> 3) ^ h) << 3) | (col & 7); }

// token order inside an 8-row half of an m-tile: {0,2,1,3,6,4,7,5}
__device__ __forceinline__ int perm8(int r) { return (0x57461320u >> (4 * r)) & 0xf; }

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
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

// word << 4 and word >> 6 as integer multiplies (IMAD / IMAD.HI), which issue
// on the FMA pipe and leave the busier integer ALU to the masks
__device__ __forceinline__ uint32_t shl4(uint32_t x) {
    uint32_t y;
    asm("mul.lo.u32 %0, %1, 16;\n" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ uint32_t shr6(uint32_t x) {
    uint32_t y;
    asm("mul.hi.u32 %0, %1, 67108864;\n" : "=r"(y) : "r"(x));
    return y;
}

// Code pair i (i = 0..7) of a 32-bit word of 16 codes -> fp16x2 subnormals
// (code_i, code_{i+8}) at mantissa bit p_i: i -> p = 4,6,4,6,8,4,6,8.
// x = word, x1 = word >> 6, x2 = word << 4.
constexpr uint32_t kM4 = 0x00300030u, kM6 = 0x00C000C0u, kM8 = 0x03000300u;
template <int I>
__device__ __forceinline__ uint32_t code_pair(uint32_t x, uint32_t x1, uint32_t x2) {
    if constexpr (I == 0) return x2 & kM4;
    else if constexpr (I == 1) return x2 & kM6;
    else if constexpr (I == 2) return x & kM4;
    else if constexpr (I == 3) return x & kM6;
    else if constexpr (I == 4) return x & kM8;
    else if constexpr (I == 5) return x1 & kM4;
    else if constexpr (I == 6) return x1 & kM6;
    else return x1 & kM8;
}
// 2^(8 - p_i) and 2^(24 - p_i)
__host__ __device__ constexpr float pair_wq(int i) {
    return (i == 4 || i == 7) ? 1.f : ((i == 1 || i == 3 || i == 6) ? 4.f : 16.f);
}
__host__ __device__ constexpr float pair_wo(int i) { return pair_wq(i) * 65536.f; }

// ---------------------------------------------------------------- partials

// Write this CTA's partial state for `unit` into slot `slot`, then let the
// last arriving CTA of the unit (S_u arrivals) merge all slots into `out`.
template <bool kMass, class A>
__device__ void finish_unit(const A &a, Smem &sm, int unit, int slot, int S_u, const float *m_h,
                            const float *l_h, const float (*y_h)[kD]) {
    const int tid = threadIdx.x;
    float *base = a.part + ((size_t)unit * a.S_max + slot) * 4 * kPartStride;
    for (int h = 0; h < a.g; ++h) {
        base[h * kPartStride + tid] = y_h[h][tid];
        if (tid == 0) {
            base[h * kPartStride + 128] = m_h[h];
            base[h * kPartStride + 129] = l_h[h];
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.flag = (atomicInc(&a.counters[unit], (unsigned)(S_u - 1)) == (unsigned)(S_u - 1));
    __syncthreads();
    if (!sm.flag) return;
    __threadfence();
    const float *ub = a.part + (size_t)unit * a.S_max * 4 * kPartStride;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int Hq = a.Hkv * a.g;
    // one pass over the unit's partials, all heads together, four slots per
    // round with every load of the round issued before any is used (online
    // rescaling: the running max moves to the larger of the two)
    float M[4], L[4], Y[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        M[h] = -INFINITY;
        L[h] = 0.f;
        Y[h] = 0.f;
    }
    for (int s0 = 0; s0 < S_u; s0 += 4) {
        float ms[4][4], ls[4][4], ys[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const bool ok = (s0 + j < S_u) && (h < a.g);
                const float *p = ub + ((s0 + j) * 4 + h) * kPartStride;
                ms[j][h] = ok ? __ldcg(p + 128) : -INFINITY;
                ls[j][h] = ok ? __ldcg(p + 129) : 0.f;
                ys[j][h] = ok ? __ldcg(p + tid) : 0.f;
            }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float m = ms[j][h], Mn = fmaxf(M[h], m);
                const float fo = (M[h] == -INFINITY) ? 0.f : ex2(M[h] - Mn);
                const float fs = (m == -INFINITY) ? 0.f : ex2(m - Mn);
                L[h] = fmaf(L[h], fo, ls[j][h] * fs);
                Y[h] = fmaf(Y[h], fo, ys[j][h] * fs);
                M[h] = Mn;
            }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h)
        if (h < a.g) {
            a.out[((size_t)b * Hq + kvh * a.g + h) * kD + tid] = f2h(__fdividef(Y[h], L[h]));
            if (kMass && tid == 0) {
                a.stats[unit * 12 + h] = M[h];
                a.stats[unit * 12 + 4 + h] = L[h];
            }
        }
    if (kMass && tid == 0) a.stats[unit * 12 + 8] = __int_as_float(len_nq(a, unit) + len_r(a, unit));
}

// Merge the four warps' states (sm.wm / wl / wy) and hand the CTA partial on.
template <bool kMass, class A>
__device__ void merge_warps_and_finish(const A &a, Smem &sm, int unit, int slot, int S_u) {
    const int tid = threadIdx.x;
    __syncthreads();
    float mh[4], lh[4], yh[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float M = fmaxf(fmaxf(sm.wm[0][h], sm.wm[1][h]), fmaxf(sm.wm[2][h], sm.wm[3][h]));
        float L = 0.f, Y = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float f = (sm.wm[w][h] == -INFINITY) ? 0.f : ex2(sm.wm[w][h] - M);
            L += f * sm.wl[w][h];
            Y += f * sm.wy[w][h][tid];
        }
        mh[h] = M;
        lh[h] = L;
        yh[h] = Y;
    }
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 4; ++h) sm.wy[0][h][tid] = yh[h];
    finish_unit<kMass>(a, sm, unit, slot, S_u, mh, lh, sm.wy[0]);
}

// packed CTA c covers slices [c*Ns/P, (c+1)*Ns/P); the CTA holding slice x
__device__ __forceinline__ int cta_of_slice(long long x, int P, int Ns) {
    return (int)(((x + 1) * P - 1) / Ns);
}
template <class A>
__device__ __forceinline__ void unit_slots(const A &a, int unit, int &first, int &S_u) {
    const int spu = len_spu(a, unit);
    if (spu == 0) {
        first = 0;
        S_u = a.n_rc;
        return;
    }
    const int s0 = slice0(a, unit);
    first = cta_of_slice(s0, part_P(a), part_Ns(a));
    const int last = cta_of_slice((long long)s0 + spu - 1, part_P(a), part_Ns(a));
    S_u = a.n_rc + last - first + 1;
}

// ------------------------------------------------------------- residual CTAs

// Residual chunk rc of a unit: logical residual tokens [64 rc, 64 rc + 64) in
// fp16; warp w takes 16 of them as one m-tile.  Scores use q (exact in fp16)
// as the B operand; outputs the same hi/lo P as the packed path.
template <bool kMass, class A>
__device__ void residual_chunk_cta(const A &a, Smem &sm, int unit, int rc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g_ = lane >> 2, t_ = lane & 3;
    const int b = unit / a.Hkv, kvh = unit % a.Hkv;
    const int Hq = a.Hkv * a.g;
    const uint16_t *knew = a.k_new + (size_t)unit * kD;
    const uint16_t *vnew = a.v_new + (size_t)unit * kD;
    uint16_t *kres = a.k_res + (size_t)unit * a.ring * kD;
    uint16_t *vres = a.v_res + (size_t)unit * a.ring * kD;
    const int r = len_r(a, unit), res_start = len_rs(a, unit), n_q = len_nq(a, unit);
    const int i0 = rc * kResChunk;
    const int n = min(kResChunk, r - i0);
    auto slot = [&](int i) { int s = res_start + i; return s >= a.ring ? s - a.ring : s; };
    auto krow = [&](int i, int c) -> const uint16_t * { return (i == r - 1 ? knew : kres + (size_t)slot(i) * kD) + c; };
    auto vrow = [&](int i, int c) -> const uint16_t * { return (i == r - 1 ? vnew : vres + (size_t)slot(i) * kD) + c; };

    {
        const int ch = tid & 15;
        int s0 = res_start + i0 + (tid >> 4);
        if (s0 >= a.ring) s0 -= a.ring;
#pragma unroll 2
        for (int row = tid >> 4; row < kResChunk; row += 8) {
            const bool ok = row < n;
            const bool newest = i0 + row == r - 1;
            const uint16_t *ks = newest ? knew : kres + (size_t)s0 * kD;
            const uint16_t *vs = newest ? vnew : vres + (size_t)s0 * kD;
            const uint32_t so = (uint32_t)swz(row, ch * 8) * 2u;
            cp_async16(smem_addr(sm.res.k) + so, (ok ? ks : kres) + ch * 8, ok);
            cp_async16(smem_addr(sm.res.v) + so, (ok ? vs : vres) + ch * 8, ok);
            s0 += 8;
            if (s0 >= a.ring) s0 -= a.ring;
        }
    }
    cp_async_commit();
    if (i0 <= r - 1 && r - 1 < i0 + n) {   // append the new token to the ring
        if (tid < 16)
            reinterpret_cast<uint4 *>(kres + (size_t)slot(r - 1) * kD)[tid] = reinterpret_cast<const uint4 *>(knew)[tid];
        else if (tid < 32)
            reinterpret_cast<uint4 *>(vres + (size_t)slot(r - 1) * kD)[tid - 16] =
                reinterpret_cast<const uint4 *>(vnew)[tid - 16];
    }
    // B operand: column g_ < 4 is query head g_ (channels in natural order), columns 4..7 are 0
    uint32_t bq[8][2];
    {
        const int hq = g_ & 3;
        const bool live = (g_ < 4) && (hq < a.g);
        const uint32_t *qp =
            reinterpret_cast<const uint32_t *>(a.q + ((size_t)b * Hq + kvh * a.g + (live ? hq : 0)) * kD);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            bq[kk][0] = live ? qp[8 * kk + t_] : 0u;
            bq[kk][1] = live ? qp[8 * kk + t_ + 4] : 0u;
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    const int hA = 2 * (t_ & 1);
    float m_w[2] = {-INFINITY, -INFINITY}, l_w[2] = {0.f, 0.f};
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    if (16 * warp < n) {
        float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t kf[4];
            ldmatrix_x4(kf, smem_addr(sm.res.k + swz(16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1),
                                                      16 * kk + 8 * (lane >> 4))));
            mma16816(s, kf, bq[kk][0], bq[kk][1]);
        }
        float x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float v = s[i] + __shfl_xor_sync(0xffffffffu, s[i], 2);
            const int row = 16 * warp + g_ + 8 * (i >> 1);
            x[i] = row < n ? v * a.scale_log2 : -INFINITY;
            if (kMass) {   // lanes t_ < 2 hold head hA + (i & 1) of token `row`
                const int h = hA + (i & 1);
                if (t_ < 2 && h < a.g && row < n)
                    a.xs[((size_t)unit * a.g + h) * a.xs_stride + n_q + i0 + row] = x[i];
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) m_w[e] = warp_max_g(fmaxf(x[e], x[e + 2]));
        uint32_t prow[2];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const float p0 = ex2(x[2 * hr] - m_w[0]), p1 = ex2(x[2 * hr + 1] - m_w[1]);
            l_w[0] += p0;
            l_w[1] += p1;
            const uint32_t hv = pack_half2(p0, p1);
            const float2 f = unpack_half2(hv);
            const uint32_t lv = pack_half2(p0 - f.x, p1 - f.y);
            prow[hr] = (t_ >= 2) ? lv : hv;
        }
        const uint32_t bv0 = movmatrix_t(prow[0]), bv1 = movmatrix_t(prow[1]);
#pragma unroll
        for (int nu = 0; nu < 8; ++nu) {
            uint32_t va[4];
            ldmatrix_x4_t(va, smem_addr(sm.res.v + swz(16 * warp + (lane & 7) + 8 * (lane >> 4),
                                                        16 * nu + 8 * ((lane >> 3) & 1))));
            mma16816(acc[nu], va, bv0, bv1);
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) l_w[e] = warp_sum_g(l_w[e]);
#pragma unroll
    for (int nu = 0; nu < 8; ++nu)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nu][i] += __shfl_xor_sync(0xffffffffu, acc[nu][i], 2);
    if (t_ < 2) {
#pragma unroll
        for (int nu = 0; nu < 8; ++nu) {
            const int ch = 16 * nu + g_;
            sm.wy[warp][hA][ch] = acc[nu][0];
            sm.wy[warp][hA + 1][ch] = acc[nu][1];
            sm.wy[warp][hA][ch + 8] = acc[nu][2];
            sm.wy[warp][hA + 1][ch + 8] = acc[nu][3];
        }
        if (g_ == 0) {
            sm.wm[warp][hA] = m_w[0];
            sm.wm[warp][hA + 1] = m_w[1];
            sm.wl[warp][hA] = l_w[0];
            sm.wl[warp][hA + 1] = l_w[1];
        }
    }
    if (r == a.ring && n_q + a.G <= a.cap && rc == 0) {
        // the oldest G residual tokens become key group n_q/G and G value tokens
        const size_t tok0 = (size_t)unit * a.cap + n_q;
        const size_t grow = (size_t)unit * (a.cap / a.G) + n_q / a.G;
        float *scr = reinterpret_cast<float *>(&sm.qn[0][0]);   // unused by residual CTAs otherwise
        if (a.G <= kResChunk) {   // the group is in this CTA's shared tile (logical rows 0..63)
            __syncthreads();
            auto kat = [&](int i, int c) -> const uint16_t * { return sm.res.k + swz(i, c); };
            auto vat = [&](int i, int c) -> const uint16_t * { return sm.res.v + swz(i, c); };
            pack_key_group(kat, a.G, a.k_codes_w + tok0 * 8, a.k_scale_w + grow * kD, a.k_zero_w + grow * kD, scr);
            pack_value_tokens(vat, a.G, kD, a.v_codes_w + tok0 * 8, a.v_scale_w + tok0, a.v_zero_w + tok0);
        } else {
            pack_key_group(krow, a.G, a.k_codes_w + tok0 * 8, a.k_scale_w + grow * kD, a.k_zero_w + grow * kD, scr);
            pack_value_tokens(vrow, a.G, kD, a.v_codes_w + tok0 * 8, a.v_scale_w + tok0, a.v_zero_w + tok0);
        }
    }
    int first, S_u;
    unit_slots(a, unit, first, S_u);
    merge_warps_and_finish<kMass>(a, sm, unit, rc, S_u);
}

// ------------------------------------------------------------------ packed CTA

// Queue the bulk copies of the slice at (unit u, slice j) into this warp's
// stage.  Called by one lane; no division: G is a power of two.
template <class A>
__device__ __forceinline__ void issue_slice(const A &a, Smem &sm, int warp, int stage, int u, int j) {
    SliceBuf &S = sm.st[warp][stage];
    uint64_t *bar = &sm.full[warp][stage];
    const int t0 = j * kSlice;
    const size_t tok = (size_t)u * a.cap + t0;
    const size_t grow = (size_t)u * a.groups_cap + (t0 >> a.lg2G);
    mbar_arrive_expect_tx(bar, kSliceBytes);
    bulk_g2s(S.kc, a.k_codes + tok * 8, kSlice * 32, bar);
    bulk_g2s(S.vc, a.v_codes + tok * 8, kSlice * 32, bar);
    bulk_g2s(S.ks, a.k_scale + grow * kD, kD * 2, bar);
    bulk_g2s(S.kz, a.k_zero + grow * kD, kD * 2, bar);
    bulk_g2s(S.vs, a.v_scale + tok, kSlice * 2, bar);
    bulk_g2s(S.vz, a.v_zero + tok, kSlice * 2, bar);
}

// A warp's position in the flat slice list, kept as (unit, its sequence b, its
// KV head kh, slice in unit j) so that stepping needs no division.
struct Cursor {
    int u, b, kh, j;
    template <class A>
    __device__ __forceinline__ void step(const A &a, int n) {
        j += n;
        int spu = seq_spu(a, b);
        while (j >= spu && u < a.units - 1) {
            j -= spu;
            ++u;
            if (++kh == a.Hkv) {
                kh = 0;
                spu = seq_spu(a, ++b);
            }
        }
    }
};

// q * 2^(8-p) for the key B operand of this lane: head g_ & 3, the channel
// pair of chunk KK, slot SIG (see code_pair)
template <int KK, int SIG>
__device__ __forceinline__ uint32_t qw_pair(const uint16_t *qh, int t_) {
    constexpr int i = 2 * (KK & 3) + SIG;
    const int c = 16 * (2 * t_ + (KK >> 2)) + i;
    constexpr float w = pair_wq(i);
    return pack_half2(h2f(qh[c]) * w, h2f(qh[c + 8]) * w);
}

// packed fp32 pairs (two lanes of work per instruction)
template <bool kMass, class A>
__device__ void packed_cta(const A &a, Smem &sm, int c) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g_ = lane >> 2, t_ = lane & 3;
    const int Hq = a.Hkv * a.g;
    const int Ns = part_Ns(a), P = part_P(a);
    if (c >= P) return;   // no share this step (device-state mode plans for the largest step)
    const int cs = (int)((long long)c * Ns / P), ce = (int)((long long)(c + 1) * Ns / P);

    if (tid == 0) {
        for (int w = 0; w < 4; ++w)
            for (int s = 0; s < kWarpStages; ++s) mbar_init(&sm.full[w][s], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // this warp's slices: cs + warp + 4k; `nxt` is the next one to queue
    Cursor nxt{0, 0, 0, 0};
    int nxt_x = cs + warp;
    if (nxt_x < ce) {
        nxt.u = unit_of(a, nxt_x);
        nxt.b = nxt.u / a.Hkv;
        nxt.kh = nxt.u - nxt.b * a.Hkv;
        nxt.j = nxt_x - slice0(a, nxt.u);
    }
    if (lane == 0)
        for (int k = 0; k < kWarpStages && nxt_x < ce; ++k) {
            issue_slice(a, sm, warp, k, nxt.u, nxt.j);
            nxt.step(a, 4);
            nxt_x += 4;
        }

    const int hA = 2 * (t_ & 1);
    const int pg = perm8(g_);
    const int p2t = perm8(2 * t_), p2t1 = perm8(2 * t_ + 1);
    const uint32_t lo_neg = (g_ >= 4) ? 0xBC00BC00u : 0u;   // fp16x2 (-1, -1) on lo columns, (0, 0) on hi
    const bool lo_row = t_ >= 2;
    int k = 0;   // this warp's slice counter over the whole range
    bool ok = true;

    int seg = cs;
    while (seg < ce) {
        const int unit = unit_of(a, seg);
        const int u_s0 = slice0(a, unit);
        const int seg_end = min(ce, u_s0 + len_spu(a, unit));
        const int b = unit / a.Hkv, kvh = unit % a.Hkv;
        const uint16_t *qbase = a.q + ((size_t)b * Hq + kvh * a.g) * kD;
        // query rows of this unit for the zero-point mma (rows >= g zero), 16-byte
        // chunks XOR-swizzled by row so the ldmatrix of 8 rows is conflict-free
        for (int e = tid; e < 8 * 16; e += kThreads) {
            const int h = e / 16, ch = e % 16;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (h < a.g) v = reinterpret_cast<const uint4 *>(qbase + (size_t)h * kD)[ch];
            *reinterpret_cast<uint4 *>(&sm.qn[h][qn_col(h, 8 * ch)]) = v;
        }
        uint32_t qw[8][2];
        {
            const int hq = g_ & 3;
            const bool live = hq < a.g;
            const uint16_t *qh = qbase + (size_t)(live ? hq : 0) * kD;
#define QW(KK)                                      \
    qw[KK][0] = live ? qw_pair<KK, 0>(qh, t_) : 0u; \
    qw[KK][1] = live ? qw_pair<KK, 1>(qh, t_) : 0u;
            QW(0) QW(1) QW(2) QW(3) QW(4) QW(5) QW(6) QW(7)
#undef QW
        }
        __syncthreads();

        // running state of heads hA, hA+1: max (log2 units), sum p, sum p*v_zero
        float m_run[2] = {-INFINITY, -INFINITY};
        unsigned long long l2 = f2pack(0.f, 0.f), pz2 = f2pack(0.f, 0.f);
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

        for (int x = cs + warp + 4 * k; ok && x < seg_end; x += 4, ++k) {
            const int stage = k % kWarpStages;
            ok = mbar_wait(&sm.full[warp][stage], (k / kWarpStages) & 1);
            if (!ok) break;
            const SliceBuf &S = sm.st[warp][stage];

            // ---- zero-point term sum_c q_c z_c: A = the key-zero row in all 16 rows
            float zc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kp = 0; kp < 4; ++kp) {
                uint32_t za[4], zb[4], qf[4];
                ldmatrix_x4(za, smem_addr(&S.kz[32 * kp + 8 * (lane >> 4)]));
                ldmatrix_x4(qf, smem_addr(&sm.qn[lane & 7][qn_col(lane & 7, 32 * kp + 8 * (lane >> 3))]));
                mma16816(zc, za, qf[0], qf[1]);
                ldmatrix_x4(zb, smem_addr(&S.kz[32 * kp + 16 + 8 * (lane >> 4)]));
                mma16816(zc, zb, qf[2], qf[3]);
            }
            // ---- scores: both m-tiles, one k-chunk at a time; B operand made just in time
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            {
                const uint2 ka0 = *reinterpret_cast<const uint2 *>(&S.kc[pg * 8 + 2 * t_]);
                const uint2 kb0 = *reinterpret_cast<const uint2 *>(&S.kc[(pg + 8) * 8 + 2 * t_]);
                const uint2 ka1 = *reinterpret_cast<const uint2 *>(&S.kc[(pg + 16) * 8 + 2 * t_]);
                const uint2 kb1 = *reinterpret_cast<const uint2 *>(&S.kc[(pg + 24) * 8 + 2 * t_]);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t a0 = half ? ka0.y : ka0.x, b0 = half ? kb0.y : kb0.x;
                    const uint32_t a1 = half ? ka1.y : ka1.x, b1 = half ? kb1.y : kb1.x;
                    const uint32_t a0r = shr6(a0), a0l = shl4(a0), b0r = shr6(b0), b0l = shl4(b0);
                    const uint32_t a1r = shr6(a1), a1l = shl4(a1), b1r = shr6(b1), b1l = shl4(b1);
#define KSTEP(Q)                                                                                               \
    {                                                                                                          \
        const int kk = 4 * half + Q;                                                                           \
        const int ch = 16 * (2 * t_ + half) + 2 * Q;                                                           \
        const uint32_t sa = *reinterpret_cast<const uint32_t *>(&S.ks[ch]);                                    \
        const uint32_t sb = *reinterpret_cast<const uint32_t *>(&S.ks[ch + 8]);                                \
        const uint32_t e0 = __byte_perm(sa, sb, 0x5410), e1 = __byte_perm(sa, sb, 0x7632);                     \
        const uint32_t bk0 = hfma2(qw[kk][0], e0, hmul2(hmul2(qw[kk][0], e0), lo_neg));                        \
        const uint32_t bk1 = hfma2(qw[kk][1], e1, hmul2(hmul2(qw[kk][1], e1), lo_neg));                        \
        const uint32_t f0[4] = {code_pair<2 * Q>(a0, a0r, a0l), code_pair<2 * Q>(b0, b0r, b0l),                \
                                code_pair<2 * Q + 1>(a0, a0r, a0l), code_pair<2 * Q + 1>(b0, b0r, b0l)};       \
        mma16816(s0, f0, bk0, bk1);                                                                            \
        const uint32_t f1[4] = {code_pair<2 * Q>(a1, a1r, a1l), code_pair<2 * Q>(b1, b1r, b1l),                \
                                code_pair<2 * Q + 1>(a1, a1r, a1l), code_pair<2 * Q + 1>(b1, b1r, b1l)};       \
        mma16816(s1, f1, bk0, bk1);                                                                            \
    }
                    KSTEP(0) KSTEP(1) KSTEP(2) KSTEP(3)
#undef KSTEP
                }
            }
            // ---- x = score * scale - mr (log2 units, relative to the running max mr;
            //      0 stands in until a first max is known)
            const float mr0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
            const float mr1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
            float x_[2][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float v0 = fmaf(zc[i], 1.f / 65536.f, s0[i]), v1 = fmaf(zc[i], 1.f / 65536.f, s1[i]);
                const float w0 = v0 + __shfl_xor_sync(0xffffffffu, v0, 2);
                const float w1 = v1 + __shfl_xor_sync(0xffffffffu, v1, 2);
                x_[0][i] = fmaf(w0, a.scale_log2 * 65536.f, (i & 1) ? -mr1 : -mr0);
                x_[1][i] = fmaf(w1, a.scale_log2 * 65536.f, (i & 1) ? -mr1 : -mr0);
            }
            if (kMass) {   // lanes t_ < 2: head hA + (i & 1), token 16 mt + 8 (i >> 1) + perm8(g_)
                const int h = hA;
                if (t_ < 2) {
                    float *xrow = a.xs + ((size_t)unit * a.g + h) * a.xs_stride + (size_t)(x - u_s0) * kSlice + pg;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (h + (i & 1) < a.g) {
                            const float ref = (i & 1) ? mr1 : mr0;
                            xrow[(i & 1) * a.xs_stride + 8 * (i >> 1)] = x_[0][i] + ref;
                            xrow[(i & 1) * a.xs_stride + 16 + 8 * (i >> 1)] = x_[1][i] + ref;
                        }
                }
            }
            // ---- online softmax: rescale only when a head's running max grows
            float mx0 = fmaxf(fmaxf(x_[0][0], x_[0][2]), fmaxf(x_[1][0], x_[1][2]));
            float mx1 = fmaxf(fmaxf(x_[0][1], x_[0][3]), fmaxf(x_[1][1], x_[1][3]));
            mx0 = warp_max_g(mx0) + mr0;   // slice max, absolute
            mx1 = warp_max_g(mx1) + mr1;
            if (__any_sync(0xffffffffu, mx0 > m_run[0] || mx1 > m_run[1])) {
                const float n0 = fmaxf(m_run[0], mx0), n1 = fmaxf(m_run[1], mx1);
                const float al0 = ex2(m_run[0] - n0), al1 = ex2(m_run[1] - n1);   // 0 on the first slice
                const float d0 = n0 - mr0, d1 = n1 - mr1;                            // shift of the reference
                m_run[0] = n0;
                m_run[1] = n1;
                l2 = fmul2(l2, f2pack(al0, al1));
                pz2 = fmul2(pz2, f2pack(al0, al1));
#pragma unroll
                for (int nu = 0; nu < 8; ++nu) {
                    acc[nu][0] *= al0;
                    acc[nu][1] *= al1;
                    acc[nu][2] *= al0;
                    acc[nu][3] *= al1;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    x_[0][i] -= (i & 1) ? d1 : d0;
                    x_[1][i] -= (i & 1) ? d1 : d0;
                }
            }
            // ---- P' = p * v_scale (hi / lo) and O^T += code^T P'
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int base = 16 * mt;
                uint32_t prow[2];
#pragma unroll
                for (int hr = 0; hr < 2; ++hr) {
                    const int tok = base + 8 * hr + pg;
                    const float vsc = h2f(S.vs[tok]), vzr = h2f(S.vz[tok]);
                    const unsigned long long p2 = f2pack(ex2(x_[mt][2 * hr]), ex2(x_[mt][2 * hr + 1]));
                    l2 = fadd2(l2, p2);
                    pz2 = ffma2(p2, f2pack(vzr, vzr), pz2);
                    const unsigned long long y2 = fmul2(p2, f2pack(vsc, vsc));
                    float y0, y1;
                    f2unpack(y2, y0, y1);
                    const uint32_t hv = pack_half2(y0, y1);
                    const float2 f = unpack_half2(hv);
                    float r0, r1;
                    f2unpack(fadd2(y2, f2pack(-f.x, -f.y)), r0, r1);
                    const uint32_t lv = pack_half2(r0, r1);
                    prow[hr] = lo_row ? lv : hv;
                }
                const uint32_t bv0 = movmatrix_t(prow[0]), bv1 = movmatrix_t(prow[1]);
                const uint32_t wA = S.vc[(base + p2t) * 8 + g_], wB = S.vc[(base + p2t1) * 8 + g_];
                const uint32_t wC = S.vc[(base + 8 + p2t) * 8 + g_], wD = S.vc[(base + 8 + p2t1) * 8 + g_];
                const uint32_t l1 = __byte_perm(wA, wB, 0x5410), h1 = __byte_perm(wA, wB, 0x7632);
                const uint32_t l2w = __byte_perm(wC, wD, 0x5410), h2 = __byte_perm(wC, wD, 0x7632);
                const uint32_t l1a = shr6(l1), l1b = shl4(l1), h1a = shr6(h1), h1b = shl4(h1);
                const uint32_t l2a = shr6(l2w), l2b = shl4(l2w), h2a = shr6(h2), h2b = shl4(h2);
#define VSTEP(NU)                                                                             \
    {                                                                                         \
        const uint32_t af[4] = {code_pair<NU>(l1, l1a, l1b), code_pair<NU>(h1, h1a, h1b),     \
                                code_pair<NU>(l2w, l2a, l2b), code_pair<NU>(h2, h2a, h2b)};   \
        mma16816(acc[NU], af, bv0, bv1);                                                      \
    }
                VSTEP(0) VSTEP(1) VSTEP(2) VSTEP(3) VSTEP(4) VSTEP(5) VSTEP(6) VSTEP(7)
#undef VSTEP
            }
            __syncwarp();
            if (lane == 0 && nxt_x < ce) {
                issue_slice(a, sm, warp, stage, nxt.u, nxt.j);
                nxt.step(a, 4);
                nxt_x += 4;
            }
        }
        if (!ok && lane == 0 && a.err) atomicExch(a.err, 1);

        // ---- warp epilogue: y[head][channel] = (O^T_hi + O^T_lo) 2^(24-p) + sum p * v_zero
        float l_run[2], pz[2];
        f2unpack(l2, l_run[0], l_run[1]);
        f2unpack(pz2, pz[0], pz[1]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            l_run[e] = warp_sum_g(l_run[e]);
            pz[e] = warp_sum_g(pz[e]);
        }
#define VOUT(NU)                                                                      \
    _Pragma("unroll") for (int i = 0; i < 4; ++i) {                                   \
        const float y = acc[NU][i] + __shfl_xor_sync(0xffffffffu, acc[NU][i], 2);     \
        acc[NU][i] = y * pair_wo(NU) + pz[i & 1];                                     \
    }
        VOUT(0) VOUT(1) VOUT(2) VOUT(3) VOUT(4) VOUT(5) VOUT(6) VOUT(7)
#undef VOUT
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
        int first, S_u;
        unit_slots(a, unit, first, S_u);
        merge_warps_and_finish<kMass>(a, sm, unit, a.n_rc + (c - first), S_u);
        seg = seg_end;
    }
}

template <bool kMass, class A>
__device__ __forceinline__ void decode_body(const A &a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw);
    // packed CTAs first: they carry most of the work; the short residual CTAs fill in behind them
    if ((int)blockIdx.x < a.P) packed_cta<kMass>(a, sm, blockIdx.x);
    else {
        const int i = blockIdx.x - a.P;
        residual_chunk_cta<kMass>(a, sm, i / a.n_rc, i % a.n_rc);
    }
}

template <bool kMass>
__global__ void __launch_bounds__(kThreads, 4) decode_kernel(const Args a) {
    decode_body<kMass>(a);
}

// Device-state mode: copy the state in, run the CTA's work, and let the last CTA
// of the launch advance the state of every sequence (append; flush G tokens
// where the ring is full).  A flush that would pass `cap` is not done: the
// sequence keeps its state and its status word is set to 1.
template <bool kMass>
__global__ void __launch_bounds__(kThreads, 4) decode_dev_kernel(const ArgsDev a) {
    const int tid = threadIdx.x;
    const int B = a.units / a.Hkv;
    int *nq = dev_arr(a, 0), *rr = dev_arr(a, 1), *rs = dev_arr(a, 2), *sbeg = dev_arr(a, 3);
    for (int b = tid; b < B; b += kThreads) {
        const int4 st = __ldcg(reinterpret_cast<const int4 *>(a.dseq) + b);
        nq[b] = st.x;
        rr[b] = st.y + 1;
        rs[b] = st.z;
    }
    __syncthreads();
    if (tid < 32) {   // sbeg = exclusive prefix of Hkv * slices, one warp, 32 sequences per pass
        int carry = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + tid;
            const int v = b < B ? a.Hkv * (nq[b] / kSlice) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (tid >= o) x += y;
            }
            if (b < B) sbeg[b] = carry + x - v;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (tid == 0) {
            sbeg[B] = carry;
            DevTab &t = dev_tab();
            t.Ns = carry;
            long long P = a.P;   // packed CTAs of the grid; at least 4 slices each
            if (P > (carry + 3) / 4) P = (carry + 3) / 4;
            t.P = (int)P;
        }
    }
    __syncthreads();
    decode_body<kMass>(a);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned n = gridDim.x;
        if (atomicInc(a.grid_counter, n - 1) == n - 1) {
            __threadfence();
            for (int b = 0; b < B; ++b) {
                int4 st = make_int4(nq[b], rr[b], rs[b], __ldcg(a.dseq + 4 * b + 3));   // status stays set
                if (rr[b] == a.ring) {
                    if (nq[b] + a.G <= a.cap) {
                        st.x += a.G;
                        st.y -= a.G;
                        st.z = (st.z + a.G) % a.ring;
                    } else {
                        st.y -= 1;   // state unchanged
                        st.w = 1;
                    }
                }
                reinterpret_cast<int4 *>(a.dseq)[b] = st;
            }
        }
    }
}

// ragged batch: per-sequence lengths in the parameter table
template <bool kMass>
__global__ void __launch_bounds__(kThreads, 4) decode_ragged_kernel(const __grid_constant__ ArgsVar a) {
    decode_body<kMass>(a);
}

// mass[unit][t] += sum_h 2^(xs[unit][h][t] - M_h) / L_h for the n_u tokens
// the unit attended to this step (n_u, M_h, L_h from the merging CTA's stats);
// grid (ceil(max n_u / 1024), units), four consecutive tokens per thread,
// all G_ score loads issued before any use.  Launched as a programmatic
// dependent of decode_kernel<true>: its launch overlaps the decode kernel's
// tail and griddepcontrol.wait holds it until that grid has finished and its
// writes are visible.  xs rows are 16-byte aligned (xs_stride4 float4s each);
// entries from n up to the row end hold no score and are never used.
template <int G_>
__global__ void __launch_bounds__(256) mass_kernel(const float4 *__restrict__ xs, const float *__restrict__ stats,
                                                   float *__restrict__ mass, int xs_stride4, long long mass_stride,
                                                   bool vec) {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    const int unit = blockIdx.y;
    const int n = __float_as_int(__ldg(stats + unit * 12 + 8));
    const int t4 = blockIdx.x * 256 + threadIdx.x;
    if (4 * t4 >= n) return;
    float4 x[G_];
#pragma unroll
    for (int h = 0; h < G_; ++h) x[h] = __ldcs(xs + (size_t)(unit * G_ + h) * xs_stride4 + t4);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int h = 0; h < G_; ++h) {
        const float M = __ldg(stats + unit * 12 + h), iL = 1.f / __ldg(stats + unit * 12 + 4 + h);
        a0 += ex2(x[h].x - M) * iL;
        a1 += ex2(x[h].y - M) * iL;
        a2 += ex2(x[h].z - M) * iL;
        a3 += ex2(x[h].w - M) * iL;
    }
    float *m = mass + (size_t)unit * mass_stride + 4 * t4;
    if (vec && 4 * t4 + 3 < n) {
        float4 v = *reinterpret_cast<float4 *>(m);
        v.x += a0;
        v.y += a1;
        v.z += a2;
        v.w += a3;
        *reinterpret_cast<float4 *>(m) = v;
    } else {
        const float a[4] = {a0, a1, a2, a3};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (4 * t4 + e < n) m[e] += a[e];
    }
}

int g_slots = 0;   // resident decode CTAs on the device (SMs x CTAs per SM)
bool g_attr_done = false;

template <class K>
bool set_smem_attr(K kernel) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(Smem)) ==
           cudaSuccess;
}

// the kernels' shared memory is above the 48 KB default: opt in once
int ensure_attr() {
    if (!g_attr_done) {
        const int dev_max = (int)(sizeof(Smem) + sizeof(DevTab) + (4 * kMaxRaggedSeqs + 1) * sizeof(int));
        if (!set_smem_attr(decode_kernel<false>) || !set_smem_attr(decode_kernel<true>) ||
            !set_smem_attr(decode_ragged_kernel<false>) || !set_smem_attr(decode_ragged_kernel<true>) ||
            cudaFuncSetAttribute(decode_dev_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dev_max) !=
                cudaSuccess ||
            cudaFuncSetAttribute(decode_dev_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, dev_max) !=
                cudaSuccess)
            return check_launch("decode_attn: cudaFuncSetAttribute");
        g_attr_done = true;
    }
    return MINIKV_OK;
}

int resident_slots() {
    if (g_slots == 0) {
        int dev = 0, sms = 148, per = 4;
        if (ensure_attr() == MINIKV_OK && cudaGetDevice(&dev) == cudaSuccess) {
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, decode_kernel<false>, kThreads, sizeof(Smem)) !=
                    cudaSuccess || per < 1)
                per = 4;
        }
        cudaGetLastError();
        g_slots = (sms > 0 ? sms : 148) * per;
    }
    return g_slots;
}

// Host state of sequence b: the table of a ragged cache, else the shared scalars.
int seq_nq(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b] : c->n_packed; }
int seq_nres(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b + 1] : c->n_res; }
int seq_rs(const minikv_cache *c, int b) { return c->seq ? c->seq[3 * b + 2] : c->res_start; }

struct Plan {
    int units, n_rc, spu, P, S_max, Ns;
    int max_n;   // most tokens any unit attends to this step
};

// shared memory of decode_dev_kernel for a batch of B sequences
size_t dev_smem_bytes(int B) { return sizeof(Smem) + sizeof(DevTab) + (4 * (size_t)B + 1) * sizeof(int); }

// resident decode_dev_kernel CTAs for this shared-memory size (looked up once
// per size, so that calls under stream capture make no occupancy query)
int dev_slots(size_t smem) {
    static size_t last_smem = 0;
    static int last_slots = 0;
    if (smem == last_smem && last_slots > 0) return last_slots;
    int dev = 0, sms = 148, per = 4;
    if (ensure_attr() == MINIKV_OK && cudaGetDevice(&dev) == cudaSuccess) {
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, decode_dev_kernel<false>, kThreads, smem) !=
                cudaSuccess || per < 1)
            per = 1;
    }
    cudaGetLastError();
    last_smem = smem;
    last_slots = (sms > 0 ? sms : 148) * per;
    return last_slots;
}

Plan plan(const minikv_cache *c) {
    Plan p;
    p.units = c->B * c->Hkv;
    if (c->dseq) {
        // device-state mode: one configuration for every state the cache can hold;
        // the kernel partitions this step's slices itself
        const int ring = c->R + c->G;
        const int spu_cap = c->cap / kSlice;
        p.n_rc = (ring + kResChunk - 1) / kResChunk;
        p.spu = 0;
        p.Ns = p.units * spu_cap;
        p.P = 0;
        if (p.Ns > 0) {
            long long P = dev_slots(dev_smem_bytes(c->B));
            if (P > (p.Ns + 3) / 4) P = (p.Ns + 3) / 4;
            if (P > kMaxPackedCtas) P = kMaxPackedCtas;
            p.P = (int)(P < 1 ? 1 : P);
        }
        int per_unit = p.Ns > 0 ? spu_cap / 3 + 2 : 0;
        if (per_unit > p.P) per_unit = p.P;
        p.S_max = p.n_rc + per_unit;
        p.max_n = c->cap + ring;
        return p;
    }
    const int nb = c->seq ? c->B : 1;   // distinct sequence states
    int max_r = 0;
    long long Ns = 0;
    p.max_n = 0;
    for (int b = 0; b < nb; ++b) {
        const int r = seq_nres(c, b) + 1;
        if (r > max_r) max_r = r;
        if (seq_nq(c, b) + r > p.max_n) p.max_n = seq_nq(c, b) + r;
        Ns += (long long)c->Hkv * (seq_nq(c, b) / kSlice);
    }
    if (!c->seq) Ns *= c->B;
    p.n_rc = (max_r + kResChunk - 1) / kResChunk;
    p.spu = c->seq ? 0 : c->n_packed / kSlice;   // slices per unit (uniform batches)
    p.Ns = (int)Ns;                             // the caller bounds units * cap / 32 below 2^31
    p.P = 0;
    if (p.Ns > 0) {
        // packed CTAs fill every resident slot, all in one wave, so that each SM
        // holds the same packed work; the short residual CTAs run as a second
        // wave behind them.  (Three of four slots, with residual CTAs mixed into
        // the first wave, measured about 10 % slower: the scheduler does not
        // spread such a mix evenly over the SMs.)
        const int slots = resident_slots();
        long long P = slots;
        const long long most = (p.Ns + 3) / 4;   // at least 4 slices per CTA
        if (P > most) P = most;
        if (P > kMaxPackedCtas) P = kMaxPackedCtas;
        if (P < 1) P = 1;
        p.P = (int)P;
    }
    // partial slots per unit: the residual chunks plus the most packed CTAs any unit meets
    int per_unit = 0;
    long long lo = 0;
    for (int u = 0; p.Ns > 0 && u < p.units; ++u) {
        const int spu = seq_nq(c, c->seq ? u / c->Hkv : 0) / kSlice;
        if (spu == 0) continue;
        const long long hi = lo + spu - 1;
        const int first = (int)(((lo + 1) * p.P - 1) / p.Ns), last = (int)(((hi + 1) * p.P - 1) / p.Ns);
        if (last - first + 1 > per_unit) per_unit = last - first + 1;
        lo = hi + 1;
    }
    p.S_max = p.n_rc + per_unit;
    return p;
}

}  // namespace

// Bytes of the workspace prefix that holds the per-unit arrival counters and
// the launch-wide counter of the device-state mode.
size_t decode_counter_bytes(int B, int Hkv) { return (((size_t)B * Hkv * 4 + 4 + 255) / 256) * 256; }

size_t decode_workspace_bytes(int B, int Hkv, int max_tokens) {
    const size_t units = (size_t)B * Hkv;
    const int res_max = max_tokens < 1024 ? max_tokens : 1024;   // the ring holds at most 1024 tokens
    const size_t n_rc = (res_max + kResChunk - 1) / kResChunk + 1;
    // every packed CTA holds at least 3 slices (the plan gives each about 4 or more)
    const size_t spu = (size_t)max_tokens / kSlice + 1;
    size_t per_unit = spu / 3 + 2;
    if (per_unit > (size_t)kMaxPackedCtas) per_unit = kMaxPackedCtas;
    return decode_counter_bytes(B, Hkv) + units * (n_rc + per_unit) * 4 * kPartStride * 4;
}

// Extra workspace of the attention-mass variant: per unit max[4], sum[4] and the
// token count, then the log2 scores of up to max_tokens tokens per unit and query head.
static size_t mass_stats_bytes(int B, int Hkv) { return (((size_t)B * Hkv * 12 * 4 + 255) / 256) * 256; }
static size_t mass_scores_bytes(int B, int Hkv, int g, int n_tokens) {
    return (size_t)B * Hkv * g * (size_t)((n_tokens + 3) & ~3) * 4;
}
size_t decode_mass_workspace_bytes(int B, int Hq, int Hkv, int max_tokens) {
    return decode_workspace_bytes(B, Hkv, max_tokens) + mass_stats_bytes(B, Hkv) +
           mass_scores_bytes(B, Hkv, Hq / Hkv, max_tokens);
}

// Workspace bytes the next decode call on this cache state will use.
size_t decode_call_workspace_bytes(const minikv_cache *c) {
    const Plan p = plan(c);
    return decode_counter_bytes(c->B, c->Hkv) + (size_t)p.units * p.S_max * 4 * kPartStride * 4;
}

namespace {

template <class A>
int launch_decode(const A &a, const Plan &p, bool with_mass, cudaStream_t stream);

template <>
int launch_decode<Args>(const Args &a, const Plan &p, bool with_mass, cudaStream_t stream) {
    const int grid = p.units * p.n_rc + p.P;
    if (with_mass) decode_kernel<true><<<grid, kThreads, sizeof(Smem), stream>>>(a);
    else decode_kernel<false><<<grid, kThreads, sizeof(Smem), stream>>>(a);
    return check_launch(with_mass ? "decode_attn_mass" : "decode_attn");
}

template <>
int launch_decode<ArgsVar>(const ArgsVar &a, const Plan &p, bool with_mass, cudaStream_t stream) {
    const int grid = p.units * p.n_rc + p.P;
    if (with_mass) decode_ragged_kernel<true><<<grid, kThreads, sizeof(Smem), stream>>>(a);
    else decode_ragged_kernel<false><<<grid, kThreads, sizeof(Smem), stream>>>(a);
    return check_launch(with_mass ? "decode_attn_mass (ragged)" : "decode_attn (ragged)");
}

template <>
int launch_decode<ArgsDev>(const ArgsDev &a, const Plan &p, bool with_mass, cudaStream_t stream) {
    const int grid = p.units * p.n_rc + p.P;
    const size_t smem = dev_smem_bytes(a.units / a.Hkv);
    if (with_mass) decode_dev_kernel<true><<<grid, kThreads, smem, stream>>>(a);
    else decode_dev_kernel<false><<<grid, kThreads, smem, stream>>>(a);
    return check_launch(with_mass ? "decode_attn_mass (device state)" : "decode_attn (device state)");
}

int launch_mass(const Args &a, const Plan &p, float *mass, long long mass_stride, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.max_n + 1023) / 1024, p.units);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float4 *xs = reinterpret_cast<const float4 *>(a.xs);
    const float *st = a.stats;
    const int xs_stride4 = a.xs_stride / 4;
    const bool vec = (mass_stride % 4 == 0) && ((reinterpret_cast<uintptr_t>(mass) & 15u) == 0);
    switch (a.g) {
        case 1: cudaLaunchKernelEx(&cfg, mass_kernel<1>, xs, st, mass, xs_stride4, mass_stride, vec); break;
        case 2: cudaLaunchKernelEx(&cfg, mass_kernel<2>, xs, st, mass, xs_stride4, mass_stride, vec); break;
        case 3: cudaLaunchKernelEx(&cfg, mass_kernel<3>, xs, st, mass, xs_stride4, mass_stride, vec); break;
        default: cudaLaunchKernelEx(&cfg, mass_kernel<4>, xs, st, mass, xs_stride4, mass_stride, vec); break;
    }
    return check_launch("decode_attn_mass: mass pass");
}

}  // namespace

int decode_launch(minikv_cache *c, const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new, int Hq,
                  float sm_scale, uint16_t *out, void *ws, size_t ws_bytes, cudaStream_t stream, float *mass) {
    const int g = Hq / c->Hkv;
    const int ring = c->R + c->G;
    const int nb = c->dseq ? 0 : (c->seq ? c->B : 1);   // device state: checked on the device
    for (int b = 0; b < nb; ++b)
        if (seq_nres(c, b) + 1 == ring && seq_nq(c, b) + c->G > c->cap)
            return fail(MINIKV_ERR_CAPACITY, "decode_attn: flushing a key group of sequence %d would exceed cap=%d",
                        b, c->cap);
    const Plan p = plan(c);
    const size_t cnt_bytes = decode_counter_bytes(c->B, c->Hkv);
    const size_t part_bytes = (size_t)p.units * p.S_max * 4 * kPartStride * 4;
    size_t need = cnt_bytes + part_bytes;
    if (mass) need += mass_stats_bytes(c->B, c->Hkv) + mass_scores_bytes(c->B, c->Hkv, g, p.max_n);
    if (ws == nullptr || ws_bytes < need)
        return fail(MINIKV_ERR_INVALID_ARG, "decode_attn: workspace of %zu bytes needed, %zu given", need, ws_bytes);
    const int arc = ensure_attr();
    if (arc) return arc;

    Args a;
    a.k_codes = c->k_codes; a.v_codes = c->v_codes;
    a.k_scale = c->k_scale; a.k_zero = c->k_zero; a.v_scale = c->v_scale; a.v_zero = c->v_zero;
    a.k_codes_w = c->k_codes; a.v_codes_w = c->v_codes;
    a.k_scale_w = c->k_scale; a.k_zero_w = c->k_zero; a.v_scale_w = c->v_scale; a.v_zero_w = c->v_zero;
    a.k_res = c->k_res; a.v_res = c->v_res;
    a.q = q; a.k_new = k_new; a.v_new = v_new; a.out = out;
    a.counters = reinterpret_cast<unsigned *>(ws);
    a.grid_counter = a.counters + p.units;
    a.dseq = c->dseq;
    a.part = reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes);
    a.err = nullptr;
    a.stats = mass ? reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes + part_bytes) : nullptr;
    a.xs = mass ? reinterpret_cast<float *>(static_cast<char *>(ws) + cnt_bytes + part_bytes +
                                            mass_stats_bytes(c->B, c->Hkv))
                : nullptr;
    a.xs_stride = (p.max_n + 3) & ~3;
    a.Hkv = c->Hkv; a.g = g; a.G = c->G; a.cap = c->cap; a.ring = ring;
    a.n_q = c->n_packed; a.r = c->n_res + 1; a.res_start = c->res_start; a.flush = (a.r == ring);
    a.groups_cap = c->cap / c->G;
    a.lg2G = 31 - __builtin_clz((unsigned)c->G);
    a.units = p.units; a.n_rc = p.n_rc; a.spu = p.spu; a.P = p.P; a.S_max = p.S_max; a.Ns = p.Ns;
    a.scale_log2 = sm_scale * kLog2e;

    int rc;
    if (c->dseq) {
        ArgsDev ad;
        static_cast<Args &>(ad) = a;
        rc = launch_decode(ad, p, mass != nullptr, stream);
        if (rc) return rc;
        return mass ? launch_mass(a, p, mass, (long long)c->cap + ring, stream) : MINIKV_OK;
    } else if (c->seq) {
        ArgsVar av;
        static_cast<Args &>(av) = a;
        av.tab.sbeg[0] = 0;
        for (int b = 0; b < c->B; ++b) {
            av.tab.n_q[b] = seq_nq(c, b);
            av.tab.r[b] = seq_nres(c, b) + 1;
            av.tab.res_start[b] = seq_rs(c, b);
            av.tab.sbeg[b + 1] = av.tab.sbeg[b] + c->Hkv * (av.tab.n_q[b] / kSlice);
        }
        rc = launch_decode(av, p, mass != nullptr, stream);
    } else {
        rc = launch_decode(a, p, mass != nullptr, stream);
    }
    if (rc) return rc;
    // host-side state: append, then flush G tokens where the ring is full
    auto advance = [&](int &n_packed, int &n_res, int &res_start) {
        n_res += 1;
        if (n_res == ring) {
            n_packed += c->G;
            n_res -= c->G;
            res_start = (res_start + c->G) % ring;
        }
    };
    if (c->seq)
        for (int b = 0; b < c->B; ++b) advance(c->seq[3 * b], c->seq[3 * b + 1], c->seq[3 * b + 2]);
    else
        advance(c->n_packed, c->n_res, c->res_start);
    return mass ? launch_mass(a, p, mass, (long long)c->cap + ring, stream) : MINIKV_OK;
}

}  // namespace minikv
